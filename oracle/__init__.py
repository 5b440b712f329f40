"""CPU oracle of the lightning indexer — test infrastructure only.

Imported only by tests/, __graft_entry__.smoke() and bench.py's CPU-baseline
and reference legs; never by the product path.  See ``oracle.indexer``.
"""
