"""CPU-side checks of the boundary: the shared library builds, loads without a
GPU, exports exactly the functions include/idx.h declares, and the binding's
signatures cover them; the product path raises when no GPU is present."""
import os
import re

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "idx.h")).read()
    return set(re.findall(r"IDX_API\s+[\w\s\*]+?\b(idx_\w+)\s*\(", src))


def test_header_declares_the_boundary():
    names = _declared()
    for n in ["idx_quant", "idx_quant_append", "idx_score", "idx_score_visible", "idx_topk", "idx_score_topk",
              "idx_workspace_size",
              "idx_status", "idx_error_string"]:
        assert n in names


def test_library_loads_and_exports_every_declared_symbol():
    from sparse_attention_token_idx_b200 import binding, build
    build.build()
    lib = binding.load()
    for n in _declared():
        assert hasattr(lib, n), n
    assert set(binding.SIGNATURES) == _declared()


def test_error_strings_without_gpu():
    from sparse_attention_token_idx_b200 import binding
    lib = binding.load()
    assert lib.idx_error_string(0) == b"ok"
    assert b"NULL" in lib.idx_error_string(-1)
    assert lib.idx_workspace_size(128, 1, 16384, 2048) == 0          # decode: selection in shared memory
    assert lib.idx_workspace_size(2, 2048, 16384, 2048) == 2 * 2048 * 16384 * 4   # prefill: fp32 score rows


def test_host_argument_checks_run_before_any_device_work():
    from sparse_attention_token_idx_b200 import binding
    lib = binding.load()
    # rejected on the host: nothing touches the (absent) GPU
    assert lib.idx_quant(None, 0, None, None, 7, None) == -3
    assert lib.idx_quant(None, 5, None, None, 0, None) == -1
    assert lib.idx_score_topk(None, None, None, None, None, 1, 1, 16, 16, 0, 0, None, None, 0, None) == -1
    assert lib.idx_topk(None, None, 1, 1, 16, 16, 0, 0, None, None, 0, None) == -4
    assert lib.idx_quant_append(None, None, -1, 1, None, None, 16, 0, None) == -2
    # the variant calls: unknown scale storage / score type, an e8m0 pitch that TMA cannot read
    p16 = 1 << 20                                   # a 16-byte aligned dummy address, never dereferenced
    assert lib.idx_score_ex(p16, p16, p16, p16, 2, p16, 1, 1, 16, 16, 0, p16, 16, 0, 0.0, None) == -3
    assert lib.idx_score_ex(p16, p16, p16, p16, 0, p16, 1, 1, 16, 16, 0, p16, 16, 5, 0.0, None) == -3
    assert lib.idx_score_ex(p16, p16, p16, p16, 1, p16, 1, 1, 20, 16, 0, p16, 16, 0, 0.0, None) == -2
    assert lib.idx_score_ex(p16, p16, p16, p16, 0, p16, 1, 1, 16, 16, 0, p16, 16, 0, float("nan"), None) == -2
    assert lib.idx_score_topk_ex(p16, p16, p16, p16, 3, p16, 1, 1, 16, 16, 0, 8, p16, None, 0, None) == -3
    assert lib.idx_quant_append_e8(None, None, 1, 1, None, None, 16, None) == -1
    # front end: unknown fmt, bad eps, nothing to do, a missing table
    assert lib.idx_front_quant_append(p16, p16, p16, p16, p16, p16, p16, 1e-6, p16, 1, 1, p16, p16, p16, p16, 16, 7,
                                      None) == -3
    assert lib.idx_front_quant_append(p16, p16, p16, p16, p16, p16, p16, float("nan"), p16, 1, 1, p16, p16, p16, p16,
                                      16, 0, None) == -2
    assert lib.idx_front_quant_append(None, None, None, None, None, None, None, 1e-6, None, 0, 1, None, None, None,
                                      None, 16, 0, None) == 0
    assert lib.idx_front_quant_append(p16, p16, p16, None, p16, p16, p16, 1e-6, p16, 1, 1, p16, p16, p16, p16, 16, 0,
                                      None) == -1
    # sparse latent attention: heads not a multiple of 16, k ≤ 0, a NaN scale, nothing to do, null
    assert lib.idx_sparse_mla_decode(p16, p16, p16, 1, 24, 16, 8, 0.1, p16, None) == -2
    assert lib.idx_sparse_mla_decode(p16, p16, p16, 1, 16, 16, 0, 0.1, p16, None) == -4
    assert lib.idx_sparse_mla_decode(p16, p16, p16, 1, 16, 16, 8, float("nan"), p16, None) == -2
    assert lib.idx_sparse_mla_decode(None, None, None, 0, 16, 16, 8, 0.1, None, None) == 0
    assert lib.idx_sparse_mla_decode(p16, None, p16, 1, 16, 16, 8, 0.1, p16, None) == -1
    # split-T calls
    assert lib.idx_gather_scores(None, 0, None, 1, 1, None, 0, None, None) == -2      # ld ≤ 0
    assert lib.idx_gather_scores(None, 16, None, 1, 1, None, 0, None, None) == -1
    assert lib.idx_gather_scores(None, 16, None, 0, 5, None, 0, None, None) == 0      # nothing to do
    assert lib.idx_merge_topk(None, 1, 1, 4, 0, None, None) == -4
    assert lib.idx_merge_topk(p16, 8, 1, 4096, 16, p16, None) == -2                  # G·kin > 16384
    assert lib.idx_merge_topk(None, 2, 1, 4, 4, None, None) == -1


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU behaviour")
def test_product_path_fails_loudly_without_gpu():
    from sparse_attention_token_idx_b200 import binding
    x = torch.zeros((4, 128), dtype=torch.bfloat16)
    with pytest.raises(binding.IdxError):
        binding.quant(x, 0)


def test_binding_shape_checks_run_on_the_host():
    """The Python wrappers of the widened calls reject inconsistent shapes
    before touching the library (CPU tensors suffice)."""
    from sparse_attention_token_idx_b200 import binding as X
    f32, i32, bf = torch.float32, torch.int32, torch.bfloat16
    with pytest.raises(ValueError):
        X.gather_scores(torch.zeros((4, 16), dtype=f32), torch.zeros((3, 8), dtype=i32), 0)
    with pytest.raises(ValueError):
        X.merge_topk(torch.zeros((2, 4, 8), dtype=i32), 8)                       # not [G, rows, kin, 2]
    with pytest.raises(ValueError):
        X.sparse_mla_decode(torch.zeros((2, 16, 512), dtype=bf), torch.zeros((2, 64, 576), dtype=bf),
                            torch.zeros((2, 8), dtype=i32), 0.1)                # 512 query features
    with pytest.raises(ValueError):
        X.sparse_mla_decode(torch.zeros((2, 16, 576), dtype=bf), torch.zeros((3, 64, 576), dtype=bf),
                            torch.zeros((2, 8), dtype=i32), 0.1)                # batch mismatch
    with pytest.raises(ValueError):
        X.front_quant_append(torch.zeros((2, 1, 64, 128), dtype=bf), torch.zeros((2, 1, 64), dtype=f32),
                             torch.zeros((2, 1, 128), dtype=bf), torch.zeros((2, 1, 16), dtype=f32),
                             torch.zeros((2, 1, 32), dtype=f32), torch.ones(128), torch.zeros(128), 1e-6,
                             torch.zeros(2, dtype=i32), torch.zeros((2, 64, 128), dtype=torch.uint8),
                             torch.zeros((2, 64), dtype=f32), 0)               # cos table of 16, not 32
