"""ctypes binding of ``libattn.so`` (C ABI in ``include/attn.h``).

Argument marshalling only: every step of the computation runs in the
library's CUDA kernels.  Importing this module loads the library and raises
``ImportError`` if it is missing; there is no CPU or PyTorch fallback.
Tensors are torch CUDA tensors used as plain device buffers.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libattn.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python -m online_softmax_12_b200.build` "
                      "(or __graft_entry__.build()); there is no fallback implementation")

_lib = ctypes.CDLL(LIB_PATH)

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_CUDA, ERR_TIMEOUT = 0, 1, 2, 3, 4
DTYPE_F32, DTYPE_BF16, DTYPE_BF16_F32OUT = 0, 1, 2
DECODE_ONE_LAUNCH = -1   # split_tokens: one kernel, clusters merge their partial states on chip

_vp, _int, _f32, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
_lib.attn_fwd.argtypes = [_vp, _vp, _vp, _vp, _vp, _int, _int, _int, _int, _int, _int, _f32, _int, _vp, _int, _vp]
_lib.attn_fwd.restype = _int
_lib.attn_decode_workspace_bytes.argtypes = [_int, _int, _int, _int, _int, _int]
_lib.attn_decode_workspace_bytes.restype = _sz
_lib.attn_decode_paged.argtypes = [_vp, _vp, _vp, _vp, _vp, _int, _int, _int, _int, _int, _int, _int, _int, _int,
                                   _f32, _vp, _sz, _vp, _vp, _vp]
_lib.attn_decode_paged.restype = _int
_lib.attn_decode_paged_static.argtypes = [_vp, _vp, _vp, _vp, _vp, _int, _int, _int, _int, _int, _int, _int,
                                          _int, _int, _f32, _vp, _vp, _vp]
_lib.attn_decode_paged_static.restype = _int
_lib.attn_fwd_fp8.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _int, _int, _int, _int, _int, _int, _f32,
                              _int, _vp, _int, _vp]
_lib.attn_fwd_fp8.restype = _int
_lib.attn_prefill_paged.argtypes = [_vp, _vp, _vp, _vp, _vp, _int, _int, _int, _int, _int, _int, _int, _int, _f32,
                                    _int, _int, _vp, _vp, _vp]
_lib.attn_prefill_paged.restype = _int
_lib.attn_bwd_workspace_bytes.argtypes = [_int, _int, _int]
_lib.attn_bwd_workspace_bytes.restype = _sz
_lib.attn_bwd.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _int, _int, _int, _int, _int, _int, _f32,
                          _int, _vp, _vp, _sz, _vp]
_lib.attn_bwd.restype = _int
_lib.attn_status_string.argtypes = [_int]
_lib.attn_status_string.restype = ctypes.c_char_p
_lib.attn_last_error.argtypes = []
_lib.attn_last_error.restype = ctypes.c_char_p
_lib.attn_check_status.argtypes = [_vp]
_lib.attn_check_status.restype = _int
_lib.attn_version.argtypes = []
_lib.attn_version.restype = _int
_lib.attn_status_detail.argtypes = [_vp]
_lib.attn_status_detail.restype = _int
_lib.attn_testing_set.argtypes = [ctypes.c_ulonglong, ctypes.c_uint]
_lib.attn_testing_set.restype = _int

# every symbol include/attn.h declares
EXPORTS = ("attn_fwd", "attn_decode_workspace_bytes", "attn_decode_paged", "attn_decode_paged_static",
           "attn_prefill_paged", "attn_fwd_fp8", "attn_bwd_workspace_bytes", "attn_bwd", "attn_status_string",
           "attn_last_error", "attn_check_status", "attn_version", "attn_status_detail")
# the test hooks include/attn_testing.h declares (not part of the product interface)
TESTING_EXPORTS = ("attn_testing_set",)
TEST_DROP_FIRST_V = 0x1


class AttnError(RuntimeError):
    def __init__(self, status: int, detail: str):
        self.status = status
        super().__init__(f"{_lib.attn_status_string(status).decode()}: {detail}")


def _check(status: int) -> None:
    if status != OK:
        raise AttnError(status, _lib.attn_last_error().decode())


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream_handle(stream, device=None):
    """The CUDA stream to launch on (the current stream when None).  The kernels run on the current
    CUDA device, so tensors on another device are refused here rather than handed over as
    foreign pointers."""
    import torch

    idx = torch.cuda.current_device()
    if device is not None and device.index != idx:
        raise ValueError(f"the tensors are on {device} but the current CUDA device is cuda:{idx}; "
                         "the kernels run on the current device (use torch.cuda.device or set_device)")
    if stream is not None:
        return ctypes.c_void_p(stream.cuda_stream)
    raw = getattr(torch._C, "_cuda_getCurrentRawStream", None)  # the handle without a Stream object
    if raw is not None:
        return ctypes.c_void_p(raw(idx))
    return ctypes.c_void_p(torch.cuda.current_stream(idx).cuda_stream)


def _expect_out(t, name, shape, dtype, device) -> None:
    """A caller-provided output must be exactly what the kernels write: a contiguous tensor
    of this shape and dtype on the inputs' device (anything else would be written out of
    bounds or through a foreign pointer)."""
    if t is None:
        return
    if t.shape != shape or t.dtype != dtype or not t.is_contiguous() or t.device != device:
        raise ValueError(f"{name} must be a contiguous {dtype} tensor of shape {tuple(shape)} on {device}; "
                         f"got {t.dtype} {tuple(t.shape)} on {t.device}"
                         f"{'' if t.is_contiguous() else ' (not contiguous)'}")


def _expect_inputs(specs, device) -> None:
    """Input tensors are handed to the kernels as raw device pointers, so each must be exactly
    what the kernels read: `specs` lists (tensor, name, dtype, shape) with None for a shape or
    dtype that is not fixed.  Shapes, dtypes and contiguity of every input are checked first,
    then that each is a CUDA tensor on `device` (a host pointer or another GPU's memory would
    fault the kernel; an int64 block table would be read as pairs of int32 page ids)."""
    for t, name, dtype, shape in specs:
        if t is None:
            continue
        if shape is not None and t.shape != shape:
            raise ValueError(f"{name} must have shape {tuple(shape)}; got {tuple(t.shape)}")
        if dtype is not None and t.dtype != dtype:
            raise ValueError(f"{name} must be {dtype}; got {t.dtype}")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    for t, name, _, _ in specs:
        if t is None:
            continue
        if not t.is_cuda or t.device != device:
            raise ValueError(f"{name} must be a CUDA tensor on {device}; got {t.device}")


def _expect_workspace(ws, need: int, device) -> int:
    """A caller-provided workspace: contiguous, on the inputs' device, at least `need` bytes.
    Returns its size in bytes."""
    nbytes = ws.numel() * ws.element_size()
    if not ws.is_contiguous() or ws.device != device or nbytes < need:
        raise ValueError(f"workspace must be a contiguous tensor of at least {need} bytes on {device}; "
                         f"got {nbytes} bytes on {ws.device}")
    return nbytes


def version() -> int:
    return int(_lib.attn_version())


def fwd_raw(q_ptr, k_ptr, v_ptr, o_ptr, lse_ptr, B, H, H_kv, n_q, n_kv, d, scale, causal, mask_ptr, dtype,
            stream_ptr) -> int:
    """Direct call with integer pointers; returns the status code."""
    return int(_lib.attn_fwd(q_ptr, k_ptr, v_ptr, o_ptr, lse_ptr, B, H, H_kv, n_q, n_kv, d, float(scale),
                             int(causal), mask_ptr, dtype, stream_ptr))


def attn_fwd(q, k, v, scale=None, causal=False, key_mask=None, o=None, lse=None, with_lse=True, stream=None,
             out_f32=False):
    """Forward attention.  q [B,H,n_q,d], k/v [B,H_kv,n_kv,d] (bf16 or fp32, contiguous, CUDA);
    key_mask [B,n_kv] uint8 or None; out_f32 writes an fp32 O for bf16 inputs.  Returns (o, lse)."""
    import torch

    B, H, n_q, d = q.shape
    _, H_kv, n_kv, _ = k.shape
    if scale is None:
        scale = d ** -0.5
    if q.dtype == torch.bfloat16:
        dt = DTYPE_BF16_F32OUT if out_f32 else DTYPE_BF16
    elif q.dtype == torch.float32:
        dt = DTYPE_F32
    else:
        raise TypeError(f"unsupported dtype {q.dtype}")
    _expect_inputs([(q, "q", q.dtype, None), (k, "k", q.dtype, (B, H_kv, n_kv, d)), (v, "v", q.dtype, k.shape),
                    (key_mask, "key_mask", torch.uint8, (B, n_kv))], q.device)
    o_dtype = torch.float32 if dt != DTYPE_BF16 else q.dtype
    if o is None:
        o = torch.empty(q.shape, dtype=o_dtype, device=q.device)
    if lse is None and with_lse:
        lse = torch.empty(B, H, n_q, dtype=torch.float32, device=q.device)
    _expect_out(o, "o", q.shape, o_dtype, q.device)
    _expect_out(lse, "lse", (B, H, n_q), torch.float32, q.device)
    _check(_lib.attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, H_kv, n_q, n_kv, d, float(scale),
                         int(bool(causal)), _ptr(key_mask), dt, _stream_handle(stream, q.device)))
    return o, lse


def _check_paged_inputs(q, k_pages, v_pages, block_table, seq_lens, S, d) -> None:
    """q bf16 with S sequences in front; K and V pools of one shape [P, page, H_kv, d] bf16; an
    int32 block table [S, max_pages] and int32 lengths [S]; all on q's CUDA device."""
    import torch

    if k_pages.dim() != 4 or k_pages.shape[3] != d:
        raise ValueError(f"k_pages must be [num_pages, page_size, H_kv, {d}]; got {tuple(k_pages.shape)}")
    if block_table.dim() != 2:
        raise ValueError(f"block_table must be [num_seqs, max_pages]; got {tuple(block_table.shape)}")
    _expect_inputs([(q, "q", torch.bfloat16, None), (k_pages, "k_pages", torch.bfloat16, None),
                    (v_pages, "v_pages", torch.bfloat16, k_pages.shape),
                    (block_table, "block_table", torch.int32, (S, block_table.shape[1])),
                    (seq_lens, "seq_lens", torch.int32, (S,))], q.device)


def decode_workspace_bytes(num_seqs, H, H_kv, d, max_seq_len, split_tokens=0) -> int:
    return int(_lib.attn_decode_workspace_bytes(num_seqs, H, H_kv, d, max_seq_len, split_tokens))


def attn_decode_paged(q, k_pages, v_pages, block_table, seq_lens, max_seq_len, scale=None, split_tokens=0,
                      workspace=None, o=None, lse=None, with_lse=True, stream=None):
    """One-token decode over a paged KV cache.  q [S,H,d] bf16; k/v_pages [P,page,H_kv,d] bf16;
    block_table [S,max_pages] int32; seq_lens [S] int32.  Returns (o, lse)."""
    import torch

    S, H, d = q.shape
    P, page, H_kv, _ = k_pages.shape
    if scale is None:
        scale = d ** -0.5
    _check_paged_inputs(q, k_pages, v_pages, block_table, seq_lens, S, d)
    need = decode_workspace_bytes(S, H, H_kv, d, max_seq_len, split_tokens)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    ws_bytes = _expect_workspace(workspace, need, q.device)
    if o is None:
        o = torch.empty_like(q)
    if lse is None and with_lse:
        lse = torch.empty(S, H, dtype=torch.float32, device=q.device)
    _expect_out(o, "o", (S, H, d), torch.bfloat16, q.device)
    _expect_out(lse, "lse", (S, H), torch.float32, q.device)
    _check(_lib.attn_decode_paged(_ptr(q), _ptr(k_pages), _ptr(v_pages), _ptr(block_table), _ptr(seq_lens), S, H,
                                  H_kv, d, page, block_table.shape[1], P, int(max_seq_len), int(split_tokens),
                                  float(scale), _ptr(workspace), ws_bytes, _ptr(o), _ptr(lse),
                                  _stream_handle(stream, q.device)))
    return o, lse


def attn_fwd_fp8(q8, k8, v8, q_descale, k_descale, v_descale, scale=None, causal=False, key_mask=None, o=None,
                 lse=None, with_lse=True, out_f32=False, stream=None):
    """Forward attention on block-scaled FP8 E4M3 inputs (uint8 bit patterns): q8 [B,H,n_q,128],
    k8/v8 [B,H_kv,n_kv,128] uint8; descales fp32 [B,H,ceil(n_q/128)] and [B,H_kv,ceil(n_kv/128)],
    one per 128-row block.  Returns (o bf16 or fp32, lse)."""
    import torch

    B, H, n_q, d = q8.shape
    _, H_kv, n_kv, _ = k8.shape
    if scale is None:
        scale = d ** -0.5
    nqb, nkb = -(-n_q // 128), -(-n_kv // 128)
    f32 = torch.float32
    _expect_inputs([(q8, "q8", torch.uint8, None), (k8, "k8", torch.uint8, (B, H_kv, n_kv, d)),
                    (v8, "v8", torch.uint8, k8.shape), (key_mask, "key_mask", torch.uint8, (B, n_kv)),
                    (q_descale, "q_descale", f32, (B, H, nqb)), (k_descale, "k_descale", f32, (B, H_kv, nkb)),
                    (v_descale, "v_descale", f32, (B, H_kv, nkb))], q8.device)
    o_dtype = torch.float32 if out_f32 else torch.bfloat16
    if o is None:
        o = torch.empty(B, H, n_q, d, dtype=o_dtype, device=q8.device)
    if lse is None and with_lse:
        lse = torch.empty(B, H, n_q, dtype=torch.float32, device=q8.device)
    _expect_out(o, "o", (B, H, n_q, d), o_dtype, q8.device)
    _expect_out(lse, "lse", (B, H, n_q), torch.float32, q8.device)
    _check(_lib.attn_fwd_fp8(_ptr(q8), _ptr(k8), _ptr(v8), _ptr(q_descale), _ptr(k_descale), _ptr(v_descale),
                             _ptr(o), _ptr(lse), B, H, H_kv, n_q, n_kv, d, float(scale), int(bool(causal)),
                             _ptr(key_mask), int(bool(out_f32)), _stream_handle(stream, q8.device)))
    return o, lse


def attn_prefill_paged(q, k_pages, v_pages, block_table, seq_lens, scale=None, causal=True, o=None, lse=None,
                       with_lse=True, stream=None, out_f32=False):
    """n_q query tokens per sequence (its last positions) over a paged KV cache.  q [S,H,n_q,d] bf16;
    k/v_pages [P,16,H_kv,d] bf16; block_table [S,max_pages] int32; seq_lens [S] int32; out_f32
    writes an fp32 O.  Returns (o, lse)."""
    import torch

    S, H, n_q, d = q.shape
    P, page, H_kv, _ = k_pages.shape
    if scale is None:
        scale = d ** -0.5
    _check_paged_inputs(q, k_pages, v_pages, block_table, seq_lens, S, d)
    o_dtype = torch.float32 if out_f32 else torch.bfloat16
    if o is None:
        o = torch.empty(q.shape, dtype=o_dtype, device=q.device)
    if lse is None and with_lse:
        lse = torch.empty(S, H, n_q, dtype=torch.float32, device=q.device)
    _expect_out(o, "o", (S, H, n_q, d), o_dtype, q.device)
    _expect_out(lse, "lse", (S, H, n_q), torch.float32, q.device)
    _check(_lib.attn_prefill_paged(_ptr(q), _ptr(k_pages), _ptr(v_pages), _ptr(block_table), _ptr(seq_lens), S, H,
                                   H_kv, n_q, d, page, block_table.shape[1], P, float(scale), int(bool(causal)),
                                   DTYPE_BF16_F32OUT if out_f32 else DTYPE_BF16, _ptr(o), _ptr(lse),
                                   _stream_handle(stream, q.device)))
    return o, lse


def attn_decode_paged_static(q, k_pages, v_pages, block_table, seq_lens, max_seq_len, scale=None, split_tokens=0,
                             o=None, lse=None, with_lse=True, stream=None):
    """attn_decode_paged with the library's fixed 32 MiB scratch instead of a workspace (no device
    allocation inside the call; o and lse are allocated here only when not given)."""
    import torch

    S, H, d = q.shape
    P, page, H_kv, _ = k_pages.shape
    if scale is None:
        scale = d ** -0.5
    _check_paged_inputs(q, k_pages, v_pages, block_table, seq_lens, S, d)
    if o is None:
        o = torch.empty_like(q)
    if lse is None and with_lse:
        lse = torch.empty(S, H, dtype=torch.float32, device=q.device)
    _expect_out(o, "o", (S, H, d), torch.bfloat16, q.device)
    _expect_out(lse, "lse", (S, H), torch.float32, q.device)
    _check(_lib.attn_decode_paged_static(_ptr(q), _ptr(k_pages), _ptr(v_pages), _ptr(block_table), _ptr(seq_lens),
                                         S, H, H_kv, d, page, block_table.shape[1], P, int(max_seq_len),
                                         int(split_tokens), float(scale), _ptr(o), _ptr(lse),
                                         _stream_handle(stream, q.device)))
    return o, lse


def check_status(stream=None) -> int:
    """Synchronise and read/clear the device status word; returns the status code."""
    return int(_lib.attn_check_status(_stream_handle(stream)))


def status_detail():
    """The four device status words (flags, first give-up site, block, parity), not cleared."""
    buf = (ctypes.c_uint * 4)()
    _check(_lib.attn_status_detail(buf))
    return list(buf)


def testing_set(wait_limit_ns: int = 0, flags: int = 0) -> None:
    """Test hook: the current device's bounded-wait limit (0 = the default 1 s) and test flags."""
    _check(_lib.attn_testing_set(int(wait_limit_ns), int(flags)))


def last_error() -> str:
    return _lib.attn_last_error().decode()


def bwd_workspace_bytes(B: int, H: int, n_q: int) -> int:
    return int(_lib.attn_bwd_workspace_bytes(B, H, n_q))


def attn_bwd(q, k, v, o, d_o, lse, scale=None, causal=False, key_mask=None, dq=None, dk=None, dv=None,
             workspace=None, stream=None):
    """Gradients of attn_fwd (bf16): q/o/d_o [B,H,n_q,d], k/v [B,H_kv,n_kv,d] contiguous bf16 CUDA
    tensors, lse [B,H,n_q] fp32 from the forward.  Returns (dq, dk, dv) as bf16 tensors."""
    import torch

    B, H, n_q, d = q.shape
    _, H_kv, n_kv, _ = k.shape
    if scale is None:
        scale = d ** -0.5
    bf = torch.bfloat16
    _expect_inputs([(q, "q", bf, None), (k, "k", bf, (B, H_kv, n_kv, d)), (v, "v", bf, k.shape),
                    (o, "o", bf, q.shape), (d_o, "d_o", bf, q.shape), (lse, "lse", torch.float32, (B, H, n_q)),
                    (key_mask, "key_mask", torch.uint8, (B, n_kv))], q.device)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    _expect_out(dq, "dq", q.shape, torch.bfloat16, q.device)
    _expect_out(dk, "dk", k.shape, torch.bfloat16, q.device)
    _expect_out(dv, "dv", v.shape, torch.bfloat16, q.device)
    need = bwd_workspace_bytes(B, H, n_q)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_bytes = _expect_workspace(workspace, need, q.device)
    _check(_lib.attn_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(d_o), _ptr(lse), _ptr(dq), _ptr(dk), _ptr(dv),
                         B, H, H_kv, n_q, n_kv, d, float(scale), int(bool(causal)), _ptr(key_mask),
                         _ptr(workspace), ws_bytes, _stream_handle(stream, q.device)))
    return dq, dk, dv
