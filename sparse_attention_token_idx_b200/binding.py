"""ctypes binding of libidx.so: argument marshalling only.

Every function here checks tensor placement, dtype and contiguity, passes raw
device pointers and the current CUDA stream to the C ABI declared in
include/idx.h, and raises on a non-zero status.  All arithmetic happens in the
library's CUDA kernels; there is no fallback path: if libidx.so is missing or
the device is not an sm_100 GPU, the calls raise.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libidx.so")

FMT_FP32 = 0
FMT_UE8M0 = 1
HEADS = 64
DIM = 128
DEV_ERR_TIMEOUT = 0x1
DEV_ERR_POSITION = 0x2
DEV_ERR_LENGTH = 0x4
SCALE_F32 = 0
SCALE_E8M0 = 1
SCORE_F32 = 0
SCORE_BF16 = 1
MASK_BOUND_BF16 = -3.3895313892515355e38    # most negative finite bfloat16

_P = ctypes.c_void_p
_I = ctypes.c_int
_I64 = ctypes.c_int64
_SZ = ctypes.c_size_t

# name → (restype, argtypes); mirrors include/idx.h
SIGNATURES = {
    "idx_quant": (_I, [_P, _I64, _P, _P, _I, _P]),
    "idx_quant_queries": (_I, [_P, _P, _I64, _P, _P, _I, _P]),
    "idx_quant_append": (_I, [_P, _P, _I, _I, _P, _P, _I, _I, _P]),
    "idx_quant_queries_append": (_I, [_P, _P, _I64, _P, _P, _P, _P, _I, _I, _P, _P, _I, _I, _P]),
    "idx_front_quant_append": (_I, [_P, _P, _P, _P, _P, _P, _P, ctypes.c_float, _P, _I, _I, _P, _P, _P, _P, _I, _I,
                                    _P]),
    "idx_quant_append_e8": (_I, [_P, _P, _I, _I, _P, _P, _I, _P]),
    "idx_score": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _P, _I64, _P]),
    "idx_score_visible": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _P, _I64, _P]),
    "idx_score_ex": (_I, [_P, _P, _P, _P, _I, _P, _I, _I, _I, _I, _I, _P, _I64, _I, ctypes.c_float, _P]),
    "idx_topk": (_I, [_P, _P, _I, _I, _I64, _I, _I, _I, _P, _P, _SZ, _P]),
    "idx_gather_scores": (_I, [_P, _I64, _P, _I64, _I, _P, _I, _P, _P]),
    "idx_merge_topk": (_I, [_P, _I, _I64, _I, _I, _P, _P]),
    "idx_sparse_mla_decode": (_I, [_P, _P, _P, _I, _I, _I64, _I, ctypes.c_float, _P, _P]),
    "idx_score_topk": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _P, _P, _SZ, _P]),
    "idx_score_topk_noalloc": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _P, _P]),
    "idx_score_topk_ex": (_I, [_P, _P, _P, _P, _I, _P, _I, _I, _I, _I, _I, _I, _P, _P, _SZ, _P]),
    "idx_workspace_size": (_SZ, [_I, _I, _I, _I]),
    "idx_project": (_I, [_P, _P, _I64, _I, _I, _P, _P, _P, _P, _P, _P, _P, _SZ, _P]),
    "idx_project_workspace_size": (_SZ, [_I64, _I, _I]),
    "idx_status": (_I, [_P]),
    "idx_device_error_bits": (ctypes.c_uint, []),
    "idx_error_string": (ctypes.c_char_p, [_I]),
    "idx_last_cuda_error": (_I, []),
    "idx_e4m3_encode": (_I, [_P, _I64, _P, _P]),
    "idx_debug_set": (None, [ctypes.c_uint, ctypes.c_ulonglong]),
    "idx_debug_trace": (_I, [_P, _I]),
}

_lib = None


class IdxError(RuntimeError):
    pass


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libidx.so (once) and declare its signatures."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise IdxError(f"{path} is missing: build it with `python -m sparse_attention_token_idx_b200.build`")
    lib = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    _lib = lib
    return lib


def _check(code: int, what: str):
    if code != 0:
        lib = load()
        msg = lib.idx_error_string(code).decode()
        raise IdxError(f"{what}: {msg} (status {code}, cuda error {lib.idx_last_cuda_error()})")


def _stream(stream=None) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _ptr(t: torch.Tensor | None, dtype=None, name="tensor") -> int | None:
    if t is None:
        return None
    if not t.is_cuda:
        raise IdxError(f"{name} must be a CUDA tensor")
    if dtype is not None and t.dtype not in (dtype if isinstance(dtype, tuple) else (dtype,)):
        raise IdxError(f"{name} has dtype {t.dtype}, expected {dtype}")
    if not t.is_contiguous():
        raise IdxError(f"{name} must be contiguous")
    return t.data_ptr()


_BF16 = (torch.bfloat16, torch.int16, torch.uint16)


def quant(x: torch.Tensor, fmt: int, out=None, scale=None, stream=None):
    """Rotate + quantise rows of 128 bf16 features → (e4m3 codes uint8, scale fp32)."""
    rows = x.numel() // DIM
    codes = out if out is not None else torch.empty(x.shape, dtype=torch.uint8, device=x.device)
    scale = scale if scale is not None else torch.empty(x.shape[:-1], dtype=torch.float32, device=x.device)
    _check(load().idx_quant(_ptr(x, _BF16, "x"), rows, _ptr(codes, torch.uint8, "out"),
                            _ptr(scale, torch.float32, "scale"), fmt, _stream(stream)), "idx_quant")
    return codes, scale


def quant_queries(q: torch.Tensor, w_raw: torch.Tensor, fmt: int, q_out=None, w_out=None, stream=None):
    """Queries [..., 64, 128] bf16 + raw head weights [..., 64] → (q codes, folded weights)."""
    tokens = q.numel() // (HEADS * DIM)
    q_out = q_out if q_out is not None else torch.empty(q.shape, dtype=torch.uint8, device=q.device)
    w_out = w_out if w_out is not None else torch.empty(w_raw.shape, dtype=torch.float32, device=q.device)
    _check(load().idx_quant_queries(_ptr(q, _BF16, "q"), _ptr(w_raw, torch.float32, "w_raw"), tokens,
                                    _ptr(q_out, torch.uint8, "q_out"), _ptr(w_out, torch.float32, "w_out"), fmt,
                                    _stream(stream)), "idx_quant_queries")
    return q_out, w_out


def quant_append(k_new: torch.Tensor, positions: torch.Tensor, k_cache: torch.Tensor,
                 k_scale_cache: torch.Tensor, fmt: int, stream=None):
    """Rotate, quantise and write k_new [B, n, 128] at slots positions[b] … (in place)."""
    B, n = k_new.shape[0], k_new.shape[1]
    T_cap = k_cache.shape[1]
    _check(load().idx_quant_append(_ptr(k_new, _BF16, "k_new"), _ptr(positions, torch.int32, "positions"), B, n,
                                   _ptr(k_cache, torch.uint8, "k_cache"),
                                   _ptr(k_scale_cache, torch.float32, "k_scale_cache"), T_cap, fmt,
                                   _stream(stream)), "idx_quant_append")


def quant_queries_append(q, w_raw, k_new, positions, k_cache, k_scale_cache, fmt, q_out, w_out, stream=None):
    """One launch: queries → (codes, folded weights) and new keys → cache slots."""
    tokens = q.numel() // (HEADS * DIM)
    B, n = k_new.shape[0], k_new.shape[1]
    _check(load().idx_quant_queries_append(
        _ptr(q, _BF16, "q"), _ptr(w_raw, torch.float32, "w_raw"), tokens, _ptr(q_out, torch.uint8, "q_out"),
        _ptr(w_out, torch.float32, "w_out"), _ptr(k_new, _BF16, "k_new"), _ptr(positions, torch.int32, "positions"),
        B, n, _ptr(k_cache, torch.uint8, "k_cache"), _ptr(k_scale_cache, torch.float32, "k_scale_cache"),
        k_cache.shape[1], fmt, _stream(stream)), "idx_quant_queries_append")
    return q_out, w_out


def front_quant_append(q_proj, w_raw, k_proj, rope_cos, rope_sin, ln_gain, ln_bias, ln_eps: float, positions,
                       k_cache, k_scale_cache, fmt, q_out=None, w_out=None, stream=None):
    """Front end + quantisation in one launch: q_proj [B, n, 64, 128] bf16 gets
    RoPE, k_proj [B, n, 128] bf16 gets LayerNorm then RoPE (cos / sin tables
    [B, n, 32] fp32, gain / bias [128] fp32); then as quant_queries_append."""
    B, n = k_proj.shape[0], k_proj.shape[1]
    q_out = q_out if q_out is not None else torch.empty(tuple(q_proj.shape), dtype=torch.uint8, device=q_proj.device)
    w_out = w_out if w_out is not None else torch.empty(tuple(w_raw.shape), dtype=torch.float32, device=q_proj.device)
    if tuple(q_proj.shape) != (B, n, HEADS, DIM) or tuple(rope_cos.shape) != (B, n, 32) or \
            tuple(rope_sin.shape) != (B, n, 32) or ln_gain.numel() != DIM or ln_bias.numel() != DIM:
        raise ValueError("front_quant_append: q_proj [B, n, 64, 128], tables [B, n, 32], gain / bias [128]")
    _check(load().idx_front_quant_append(
        _ptr(q_proj, _BF16, "q_proj"), _ptr(w_raw, torch.float32, "w_raw"), _ptr(k_proj, _BF16, "k_proj"),
        _ptr(rope_cos, torch.float32, "rope_cos"), _ptr(rope_sin, torch.float32, "rope_sin"),
        _ptr(ln_gain, torch.float32, "ln_gain"), _ptr(ln_bias, torch.float32, "ln_bias"), float(ln_eps),
        _ptr(positions, torch.int32, "positions"), B, n, _ptr(q_out, torch.uint8, "q_out"),
        _ptr(w_out, torch.float32, "w_out"), _ptr(k_cache, torch.uint8, "k_cache"),
        _ptr(k_scale_cache, torch.float32, "k_scale_cache"), k_cache.shape[1], fmt, _stream(stream)),
        "idx_front_quant_append")
    return q_out, w_out


def project_workspace_size(tokens: int, hidden: int, q_lora: int) -> int:
    return int(load().idx_project_workspace_size(tokens, hidden, q_lora))


def project(x, qr, wq_b, wk, w_proj, q_out=None, k_out=None, w_out=None, ws=None, stream=None):
    """The three projections: x [T, hidden] bf16, qr [T, q_lora] bf16, wq_b
    [64·128, q_lora] bf16, wk [128, hidden] bf16, w_proj [64, hidden] fp32 →
    (q_proj [T, 64, 128] bf16, k_proj [T, 128] bf16, w_raw [T, 64] fp32).
    ws: uint8 workspace of project_workspace_size bytes (allocated when None)."""
    T, hidden = x.shape
    q_lora = qr.shape[1]
    if tuple(qr.shape) != (T, q_lora) or tuple(wq_b.shape) != (HEADS * DIM, q_lora) or \
            tuple(wk.shape) != (DIM, hidden) or tuple(w_proj.shape) != (HEADS, hidden):
        raise ValueError("project: x [T, hidden], qr [T, q_lora], wq_b [8192, q_lora], wk [128, hidden], "
                         "w_proj [64, hidden]")
    dev = x.device
    q_out = q_out if q_out is not None else torch.empty((T, HEADS, DIM), dtype=torch.bfloat16, device=dev)
    k_out = k_out if k_out is not None else torch.empty((T, DIM), dtype=torch.bfloat16, device=dev)
    w_out = w_out if w_out is not None else torch.empty((T, HEADS), dtype=torch.float32, device=dev)
    need = project_workspace_size(T, hidden, q_lora)
    if ws is None and need:
        ws = torch.empty(need, dtype=torch.uint8, device=dev)
    _check(load().idx_project(
        _ptr(x, _BF16, "x"), _ptr(qr, _BF16, "qr"), T, hidden, q_lora, _ptr(wq_b, _BF16, "wq_b"),
        _ptr(wk, _BF16, "wk"), _ptr(w_proj, torch.float32, "w_proj"), _ptr(q_out, _BF16, "q_out"),
        _ptr(k_out, _BF16, "k_out"), _ptr(w_out, torch.float32, "w_out"),
        _ptr(ws, torch.uint8, "ws") if ws is not None else None, ws.numel() if ws is not None else 0,
        _stream(stream)), "idx_project")
    return q_out, k_out, w_out


def score(q_fp8, w, k_cache, k_scale_cache, lengths, causal: bool, max_len: int, ld: int | None = None,
          out=None, stream=None):
    """Scores [B, n, ld] fp32 (−inf outside each row's visible keys)."""
    B, n = q_fp8.shape[0], q_fp8.shape[1]
    T_cap = k_cache.shape[1]
    ld = ld if ld is not None else max_len
    out = out if out is not None else torch.empty((B, n, ld), dtype=torch.float32, device=q_fp8.device)
    _check(load().idx_score(_ptr(q_fp8, torch.uint8, "q_fp8"), _ptr(w, torch.float32, "w"),
                            _ptr(k_cache, torch.uint8, "k_cache"), _ptr(k_scale_cache, torch.float32, "k_scale"),
                            _ptr(lengths, torch.int32, "lengths"), B, n, T_cap, max_len, int(causal),
                            _ptr(out, torch.float32, "scores"), ld, _stream(stream)), "idx_score")
    return out


def score_visible(q_fp8, w, k_cache, k_scale_cache, lengths, causal: bool, max_len: int, ld: int | None = None,
                  out=None, stream=None):
    """Scores [B, n, ld] fp32 of the visible keys (−inf up to the end of each row's
    last 128-key tile, later columns unwritten): the workspace the score + top-k
    path fills."""
    B, n = q_fp8.shape[0], q_fp8.shape[1]
    T_cap = k_cache.shape[1]
    ld = ld if ld is not None else max_len
    out = out if out is not None else torch.empty((B, n, ld), dtype=torch.float32, device=q_fp8.device)
    _check(load().idx_score_visible(_ptr(q_fp8, torch.uint8, "q_fp8"), _ptr(w, torch.float32, "w"),
                                    _ptr(k_cache, torch.uint8, "k_cache"),
                                    _ptr(k_scale_cache, torch.float32, "k_scale"),
                                    _ptr(lengths, torch.int32, "lengths"), B, n, T_cap, max_len, int(causal),
                                    _ptr(out, torch.float32, "scores"), ld, _stream(stream)), "idx_score_visible")
    return out


def quant_append_e8(k_new, positions, k_cache, k_scale_e8, stream=None):
    """Rotate, quantise (ue8m0) and append keys; scales stored as e8m0 bytes."""
    B, n = k_new.shape[0], k_new.shape[1]
    _check(load().idx_quant_append_e8(_ptr(k_new, _BF16, "k_new"), _ptr(positions, torch.int32, "positions"),
                                      B, n, _ptr(k_cache, torch.uint8, "k_cache"),
                                      _ptr(k_scale_e8, torch.uint8, "k_scale_e8"), k_cache.shape[1],
                                      _stream(stream)), "idx_quant_append_e8")


def _scale_arg(k_scale):
    if k_scale.dtype == torch.uint8:
        return _ptr(k_scale, torch.uint8, "k_scale"), SCALE_E8M0
    return _ptr(k_scale, torch.float32, "k_scale"), SCALE_F32


def score_ex(q_fp8, w, k_cache, k_scale, lengths, causal: bool, max_len: int, ld: int | None = None,
             dtype=torch.float32, mask_value: float = float("-inf"), out=None, stream=None):
    """Scores [B, n, ld] in fp32 or bf16 with a chosen mask value; key scales fp32
    or e8m0 bytes (uint8)."""
    B, n = q_fp8.shape[0], q_fp8.shape[1]
    T_cap = k_cache.shape[1]
    ld = ld if ld is not None else max_len
    out = out if out is not None else torch.empty((B, n, ld), dtype=dtype, device=q_fp8.device)
    sdt = SCORE_BF16 if out.dtype == torch.bfloat16 else SCORE_F32
    ks, sfmt = _scale_arg(k_scale)
    _check(load().idx_score_ex(_ptr(q_fp8, torch.uint8, "q_fp8"), _ptr(w, torch.float32, "w"),
                               _ptr(k_cache, torch.uint8, "k_cache"), ks, sfmt, _ptr(lengths, torch.int32, "lengths"),
                               B, n, T_cap, max_len, int(causal), _ptr(out, out.dtype, "scores"), ld, sdt,
                               float(mask_value), _stream(stream)), "idx_score_ex")
    return out


def score_topk_ex(q_fp8, w, k_cache, k_scale, lengths, causal: bool, k: int, max_len: int, out=None,
                  ws: torch.Tensor | None = None, stream=None):
    """score_topk with key scales fp32 or e8m0 bytes (uint8)."""
    B, n = q_fp8.shape[0], q_fp8.shape[1]
    out = out if out is not None else torch.empty((B, n, k), dtype=torch.int32, device=q_fp8.device)
    ks, sfmt = _scale_arg(k_scale)
    wsp, wsn = (None, 0) if ws is None else (_ptr(ws, None, "ws"), ws.numel() * ws.element_size())
    _check(load().idx_score_topk_ex(_ptr(q_fp8, torch.uint8, "q_fp8"), _ptr(w, torch.float32, "w"),
                                    _ptr(k_cache, torch.uint8, "k_cache"), ks, sfmt,
                                    _ptr(lengths, torch.int32, "lengths"), B, n, k_cache.shape[1], max_len,
                                    int(causal), k, _ptr(out, torch.int32, "indices"), wsp, wsn, _stream(stream)),
           "idx_score_topk_ex")
    return out


def gather_scores(scores, idx, offset: int, counts=None, out=None, stream=None):
    """(score, global position) pairs of a slice's top-k: scores [rows, ld] fp32,
    idx [rows, k] int32 slice-local (−1 empty), counts [rows] int32 keys held per
    row (None: all) → int32 [rows, k, 2] holding idx_cand_t pairs (score bits,
    position); (−inf, −1) for empty slots."""
    rows, ld = scores.shape
    k = idx.shape[-1]
    if tuple(idx.shape) != (rows, k):
        raise ValueError("gather_scores: scores [rows, ld], idx [rows, k]")
    out = out if out is not None else torch.empty((rows, k, 2), dtype=torch.int32, device=scores.device)
    if tuple(out.shape[-3:]) != (rows, k, 2):
        raise ValueError("gather_scores: out [rows, k, 2] int32")
    _check(load().idx_gather_scores(_ptr(scores, torch.float32, "scores"), ld, _ptr(idx, torch.int32, "idx"), rows, k,
                                    _ptr(counts, torch.int32, "counts"), int(offset), _ptr(out, torch.int32, "cand"),
                                    _stream(stream)),
           "idx_gather_scores")
    return out


def cand_scores(cand: torch.Tensor) -> torch.Tensor:
    """The score plane of idx_cand_t pairs (int32 [..., 2]) as float32 [...]."""
    return cand.view(torch.float32)[..., 0]


def merge_topk(cand, k: int, out=None, stream=None):
    """Top-k positions [rows, k] int32 among candidates int32 [G, rows, kin, 2]
    (idx_cand_t pairs; position −1 = empty)."""
    if cand.dim() != 4 or cand.shape[-1] != 2:
        raise ValueError("merge_topk: cand int32 [G, rows, kin, 2]")
    G, rows, kin, _ = cand.shape
    out = out if out is not None else torch.empty((rows, k), dtype=torch.int32, device=cand.device)
    _check(load().idx_merge_topk(_ptr(cand, torch.int32, "cand"), G, rows, kin, k, _ptr(out, torch.int32, "out"),
                                 _stream(stream)), "idx_merge_topk")
    return out


def sparse_mla_decode(q, kv, indices, softmax_scale: float, out=None, stream=None):
    """Latent output [B, H, 512] fp32 of one decode token per sequence attending
    over its selected positions: q [B, H, 576] bf16, kv [B, T_cap, 576] bf16,
    indices [B, k] int32 (−1 = none)."""
    B, H, D = q.shape
    if D != 576 or kv.dim() != 3 or kv.shape[0] != B or kv.shape[2] != 576 or indices.dim() != 2 or \
            indices.shape[0] != B:
        raise ValueError("sparse_mla_decode: q [B, H, 576], kv [B, T_cap, 576], indices [B, k]")
    out = out if out is not None else torch.empty((B, H, 512), dtype=torch.float32, device=q.device)
    _check(load().idx_sparse_mla_decode(_ptr(q, _BF16, "q"), _ptr(kv, _BF16, "kv"), _ptr(indices, torch.int32, "indices"),
                                        B, H, kv.shape[1], indices.shape[1], float(softmax_scale),
                                        _ptr(out, torch.float32, "out"), _stream(stream)), "idx_sparse_mla_decode")
    return out


def topk(scores, lengths, causal: bool, k: int, max_len: int, out=None, stream=None):
    """Top-k positions [B, n, k] int32 (a set per row, −1 padded) of materialised scores [B, n, ld]."""
    B, n, ld = scores.shape
    out = out if out is not None else torch.empty((B, n, k), dtype=torch.int32, device=scores.device)
    _check(load().idx_topk(_ptr(scores, torch.float32, "scores"), _ptr(lengths, torch.int32, "lengths"), B, n, ld,
                           max_len, int(causal), k, _ptr(out, torch.int32, "indices"), None, 0, _stream(stream)),
           "idx_topk")
    return out


def workspace_size(B: int, n: int, max_len: int, k: int) -> int:
    return int(load().idx_workspace_size(B, n, max_len, k))


def score_topk(q_fp8, w, k_cache, k_scale_cache, lengths, causal: bool, k: int, max_len: int, out=None,
               ws: torch.Tensor | None = None, stream=None):
    """Scores + top-k: positions [B, n, k] int32 (a set per row, −1 padded).
    ``ws`` (a uint8 CUDA tensor of workspace_size() bytes) is used by
    prefill-shaped calls; decode-shaped calls need none."""
    B, n = q_fp8.shape[0], q_fp8.shape[1]
    T_cap = k_cache.shape[1]
    out = out if out is not None else torch.empty((B, n, k), dtype=torch.int32, device=q_fp8.device)
    ws_ptr, ws_bytes = (None, 0) if ws is None else (_ptr(ws, None, "ws"), ws.numel() * ws.element_size())
    _check(load().idx_score_topk(_ptr(q_fp8, torch.uint8, "q_fp8"), _ptr(w, torch.float32, "w"),
                                 _ptr(k_cache, torch.uint8, "k_cache"),
                                 _ptr(k_scale_cache, torch.float32, "k_scale"),
                                 _ptr(lengths, torch.int32, "lengths"), B, n, T_cap, max_len, int(causal), k,
                                 _ptr(out, torch.int32, "indices"), ws_ptr, ws_bytes, _stream(stream)),
           "idx_score_topk")
    return out


def e4m3_encode(x: torch.Tensor, stream=None) -> torch.Tensor:
    out = torch.empty(x.shape, dtype=torch.uint8, device=x.device)
    _check(load().idx_e4m3_encode(_ptr(x, torch.float32, "x"), x.numel(), _ptr(out, torch.uint8, "out"),
                                  _stream(stream)), "idx_e4m3_encode")
    return out


def status(stream=None) -> tuple[int, int]:
    """(status code, device error bits); synchronises the stream and clears the device error word."""
    lib = load()
    code = lib.idx_status(_stream(stream))
    return code, int(lib.idx_device_error_bits())


def debug_set(flags: int, budget_ns: int = 0):
    load().idx_debug_set(flags, budget_ns)


def debug_trace(max_ctas: int):
    """Per-CTA phase timestamps of the last traced score launch (see include/idx.h)."""
    import numpy as np
    buf = np.zeros((max_ctas, 16), np.uint64)
    _check(load().idx_debug_trace(buf.ctypes.data, max_ctas), "idx_debug_trace")
    return buf
