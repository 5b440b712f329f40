"""B200 (sm_100a) lightning indexer: rotate + FP8-quantise + append keys,
score FP8 queries against the FP8 key cache, select the top-k positions.

The compute lives in libidx.so (CUDA, C ABI in include/idx.h); ``binding``
marshals torch tensors into it.  ``synth`` draws seeded synthetic inputs.
Submodules are imported on demand so that the input generator can be used
without the CUDA library.
"""
__all__ = ["binding", "synth", "build", "parallel"]
