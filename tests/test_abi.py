"""The C-ABI library builds, loads, exports every declared symbol, and rejects
bad arguments on the host before any launch (no GPU needed for any of this)."""
import ctypes
import os
import re

import pytest

from conftest import ROOT

HEADER = os.path.join(ROOT, "include", "attn.h")
TESTING_HEADER = os.path.join(ROOT, "include", "attn_testing.h")


def _lib():
    from online_softmax_12_b200 import build

    build.build()
    from online_softmax_12_b200 import attn

    return attn


def _declared(path=HEADER):
    text = open(path).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(attn_[a-z_0-9]+)\s*\(", text)))


def test_every_declared_symbol_is_exported():
    attn = _lib()
    declared = _declared()
    assert declared, "no declarations found"
    lib = ctypes.CDLL(attn.LIB_PATH)
    for name in declared:
        assert hasattr(lib, name), f"{name} declared in attn.h but not exported"
    assert sorted(attn.EXPORTS) == declared
    testing = _declared(TESTING_HEADER)
    assert testing == sorted(attn.TESTING_EXPORTS)
    for name in testing:
        assert hasattr(lib, name), f"{name} declared in attn_testing.h but not exported"
    # every header under include/ is one of the two
    assert sorted(os.listdir(os.path.join(ROOT, "include"))) == ["attn.h", "attn_testing.h"]


def test_testing_hook_rejects_unknown_flags():
    attn = _lib()
    assert attn._lib.attn_testing_set(0, 0x80) == attn.ERR_INVALID_ARG
    assert "test flags" in attn.last_error()


def test_binding_loads_the_in_tree_library():
    attn = _lib()
    assert os.path.dirname(attn.LIB_PATH) == os.path.join(ROOT, "online_softmax_12_b200")
    assert attn.version() == 10000
    assert attn._lib.attn_status_string(attn.ERR_TIMEOUT).decode().startswith("a bounded wait")


@pytest.mark.parametrize("args, status, needle", [
    (dict(H=3, H_kv=2), 1, "multiple of H_kv"),
    (dict(d=80), 2, "head dim"),
    (dict(scale=-1.0), 2, "scale"),
    (dict(scale=float("nan")), 2, "scale"),
    (dict(causal=2), 1, "causal"),
    (dict(B=0), 1, "positive"),
    (dict(q=0), 1, "null"),
    (dict(q=0x1008), 1, "aligned"),
])
def test_forward_rejects_bad_arguments_before_launch(args, status, needle):
    attn = _lib()
    a = dict(q=0x1000, k=0x2000, v=0x3000, o=0x4000, lse=None, B=1, H=2, H_kv=2, n_q=4, n_kv=4, d=64, scale=0.125,
             causal=0, mask=None, dtype=attn.DTYPE_BF16, stream=None)
    a.update(args)
    st = attn.fwd_raw(a["q"], a["k"], a["v"], a["o"], a["lse"], a["B"], a["H"], a["H_kv"], a["n_q"], a["n_kv"],
                      a["d"], a["scale"], a["causal"], a["mask"], a["dtype"], a["stream"])
    assert st == status
    assert needle in attn.last_error()


def test_empty_query_is_a_noop():
    attn = _lib()
    assert attn.fwd_raw(None, None, None, None, None, 1, 1, 1, 0, 5, 64, 0.1, 0, None, attn.DTYPE_BF16, None) == 0


def test_decode_workspace_size_and_validation():
    attn = _lib()
    # 64 sequences, 32 heads, d = 128, up to 8192 tokens, 512-token splits: 16 splits of
    # (m, l, l, pad) + u per head
    n = attn.decode_workspace_bytes(64, 32, 8, 128, 8192, 512)
    slots = 64 * 32 * 16
    assert n >= slots * (4 + 128) * 4 and n < slots * (4 + 128) * 4 + 1024
    # the default for 64 sequences x 8 kv heads up to 8192 tokens: 1024-token splits
    assert attn.decode_workspace_bytes(64, 32, 8, 128, 8192, 0) == attn.decode_workspace_bytes(64, 32, 8, 128, 8192, 1024)
    assert attn.decode_workspace_bytes(64, 32, 8, 128, 8192, 1024) < n
    assert attn.decode_workspace_bytes(-1, 32, 8, 128, 8192, 0) == 0
    lib = attn._lib
    # G = 3 unsupported, d = 96 unsupported, workspace too small
    st = lib.attn_decode_paged(0x1000, 0x2000, 0x3000, 0x4000, 0x5000, 2, 6, 2, 128, 16, 4, 8, 64, 0, 0.1,
                               0x6000, 1 << 30, 0x7000, None, None)
    assert st == attn.ERR_UNSUPPORTED
    st = lib.attn_decode_paged(0x1000, 0x2000, 0x3000, 0x4000, 0x5000, 2, 8, 2, 96, 16, 4, 8, 64, 0, 0.1,
                               0x6000, 1 << 30, 0x7000, None, None)
    assert st == attn.ERR_UNSUPPORTED
    st = lib.attn_decode_paged(0x1000, 0x2000, 0x3000, 0x4000, 0x5000, 2, 8, 2, 128, 16, 4, 8, 64, 0, 0.1,
                               0x6000, 16, 0x7000, None, None)
    assert st == attn.ERR_INVALID_ARG and "workspace" in attn.last_error()
    st = lib.attn_decode_paged(0x1000, 0x2000, 0x3000, 0x4000, 0x5000, 2, 8, 2, 128, 16, 4, 8, 65, 0, 0.1,
                               0x6000, 1 << 30, 0x7000, None, None)
    assert st == attn.ERR_INVALID_ARG  # max_seq_len beyond max_pages * page_size
    # the single launch: 16-token pages only, no workspace needed; split_tokens below -1 is invalid
    assert attn.decode_workspace_bytes(64, 32, 8, 128, 8192, attn.DECODE_ONE_LAUNCH) == 16
    st = lib.attn_decode_paged(0x1000, 0x2000, 0x3000, 0x4000, 0x5000, 2, 8, 2, 128, 8, 8, 8, 64,
                               attn.DECODE_ONE_LAUNCH, 0.1, None, 0, 0x7000, None, None)
    assert st == attn.ERR_UNSUPPORTED and "16-token pages" in attn.last_error()
    st = lib.attn_decode_paged(0x1000, 0x2000, 0x3000, 0x4000, 0x5000, 2, 8, 2, 128, 16, 4, 8, 64, -2, 0.1,
                               0x6000, 1 << 30, 0x7000, None, None)
    assert st == attn.ERR_INVALID_ARG


def test_paged_prefill_rejects_bad_arguments_before_launch():
    attn = _lib()
    lib = attn._lib
    args = dict(q=0x1000, k=0x2000, v=0x3000, bt=0x4000, sl=0x5000, S=2, H=8, H_kv=2, n_q=64, d=128, page=16,
                max_pages=8, pages=32, scale=0.1, causal=1, dtype=attn.DTYPE_BF16, o=0x6000, lse=None)

    def call(**kw):
        a = dict(args)
        a.update(kw)
        return lib.attn_prefill_paged(a["q"], a["k"], a["v"], a["bt"], a["sl"], a["S"], a["H"], a["H_kv"], a["n_q"],
                                      a["d"], a["page"], a["max_pages"], a["pages"], a["scale"], a["causal"],
                                      a["dtype"], a["o"], a["lse"], None)

    assert call(page=8) == attn.ERR_UNSUPPORTED and "16-token pages" in attn.last_error()
    assert call(d=96) == attn.ERR_UNSUPPORTED
    assert call(H=6, H_kv=4) == attn.ERR_INVALID_ARG
    assert call(causal=3) == attn.ERR_INVALID_ARG
    assert call(dtype=attn.DTYPE_F32) == attn.ERR_INVALID_ARG and "dtype" in attn.last_error()
    assert call(scale=0.0) == attn.ERR_UNSUPPORTED
    assert call(bt=0) == attn.ERR_INVALID_ARG and "null" in attn.last_error()
    assert call(q=0x1008) == attn.ERR_INVALID_ARG and "misaligned" in attn.last_error()
    assert call(n_q=0, q=0, o=0) == attn.OK   # nothing to do
    assert call(S=0) == attn.OK


def test_backward_workspace_and_validation():
    attn = _lib()
    lib = attn._lib
    # two fp32 values per query row, rows padded to 64 per head, each array 256-byte aligned
    assert attn.bwd_workspace_bytes(1, 32, 16384) == 2 * 32 * 16384 * 4
    assert attn.bwd_workspace_bytes(2, 3, 65) == 2 * (((2 * 3 * 128 * 4) + 255) // 256 * 256)
    assert attn.bwd_workspace_bytes(0, 3, 65) == 0
    args = dict(q=0x1000, k=0x2000, v=0x3000, o=0x4000, do=0x5000, lse=0x6000, dq=0x7000, dk=0x8000, dv=0x9000,
                B=1, H=8, H_kv=2, n_q=100, n_kv=100, d=128, scale=0.1, causal=1, mask=None, ws=0x10000,
                ws_bytes=1 << 20)

    def call(**kw):
        a = dict(args)
        a.update(kw)
        return lib.attn_bwd(a["q"], a["k"], a["v"], a["o"], a["do"], a["lse"], a["dq"], a["dk"], a["dv"], a["B"],
                            a["H"], a["H_kv"], a["n_q"], a["n_kv"], a["d"], a["scale"], a["causal"], a["mask"],
                            a["ws"], a["ws_bytes"], None)

    assert call(d=96) == attn.ERR_UNSUPPORTED and "head dim" in attn.last_error()
    assert call(H=6, H_kv=4) == attn.ERR_INVALID_ARG
    assert call(causal=2) == attn.ERR_INVALID_ARG
    assert call(scale=float("inf")) == attn.ERR_UNSUPPORTED
    assert call(do=0) == attn.ERR_INVALID_ARG and "null" in attn.last_error()
    assert call(lse=0) == attn.ERR_INVALID_ARG
    assert call(dk=0x8008) == attn.ERR_INVALID_ARG and "aligned" in attn.last_error()
    assert call(ws_bytes=16) == attn.ERR_INVALID_ARG and "workspace" in attn.last_error()
    assert call(ws=0x10010) == attn.ERR_INVALID_ARG and "workspace" in attn.last_error()
    assert call(B=-1) == attn.ERR_INVALID_ARG
    assert call(n_q=0, n_kv=0) == attn.OK   # no gradient exists: nothing to write


def test_binding_rejects_mismatched_outputs_and_workspaces():
    import torch

    attn = _lib()
    cpu = torch.device("cpu")
    ok = torch.empty(2, 3, 4, dtype=torch.bfloat16)
    attn._expect_out(ok, "o", (2, 3, 4), torch.bfloat16, cpu)
    attn._expect_out(None, "lse", (2, 3), torch.float32, cpu)   # not given: allocated by the binding
    for bad in (torch.empty(2, 3, 5, dtype=torch.bfloat16),          # shape
                torch.empty(2, 3, 4, dtype=torch.float32),           # dtype
                torch.empty(2, 4, 3, dtype=torch.bfloat16).transpose(1, 2)):   # not contiguous
        with pytest.raises(ValueError):
            attn._expect_out(bad, "o", (2, 3, 4), torch.bfloat16, cpu)
    with pytest.raises(ValueError):
        attn._expect_out(ok, "o", (2, 3, 4), torch.bfloat16, torch.device("meta"))   # another device
    assert attn._expect_workspace(torch.empty(64, dtype=torch.float32), 256, cpu) == 256
    with pytest.raises(ValueError):
        attn._expect_workspace(torch.empty(63, dtype=torch.float32), 256, cpu)        # too small
    with pytest.raises(ValueError):
        attn._expect_workspace(torch.empty(512, dtype=torch.uint8)[::2], 256, cpu)    # strided


def test_binding_rejects_mismatched_inputs_before_the_call():
    """Every input reaches the kernels as a raw device pointer, so the binding checks
    shape, dtype, contiguity and device of each before calling the library: an int64
    block table, a V pool smaller than the K pool, a host tensor or a strided tensor
    must raise instead of reaching a kernel."""
    import torch

    attn = _lib()
    S, H, H_kv, d, P = 2, 4, 2, 64, 6
    q = torch.zeros(S, H, d, dtype=torch.bfloat16)
    kp = torch.zeros(P, 16, H_kv, d, dtype=torch.bfloat16)
    bt = torch.zeros(S, 3, dtype=torch.int32)
    sl = torch.zeros(S, dtype=torch.int32)
    cases = [
        (dict(block_table=bt.to(torch.int64)), "block_table must be torch.int32"),
        (dict(seq_lens=sl.to(torch.int64)), "seq_lens must be torch.int32"),
        (dict(v_pages=kp[: P - 1].clone()), "v_pages must have shape"),
        (dict(seq_lens=torch.zeros(S + 1, dtype=torch.int32)), "seq_lens must have shape"),
        (dict(block_table=torch.zeros(S + 1, 3, dtype=torch.int32)), "block_table must have shape"),
        (dict(q=q.float()), "q must be torch.bfloat16"),
        (dict(k_pages=torch.zeros(P, 16, H_kv, 2 * d, dtype=torch.bfloat16)[..., ::2]), "k_pages must be contiguous"),
        (dict(), "must be a CUDA tensor"),          # everything consistent, but on the host
    ]
    for over, needle in cases:
        a = dict(q=q, k_pages=kp, v_pages=kp.clone(), block_table=bt, seq_lens=sl)
        a.update(over)
        for fn in (attn.attn_decode_paged, attn.attn_decode_paged_static):
            with pytest.raises(ValueError, match=needle):
                fn(a["q"], a["k_pages"], a["v_pages"], a["block_table"], a["seq_lens"], 48)
        qp = a["q"][:, :, None, :].expand(S, H, 5, a["q"].shape[-1]).contiguous()
        if "q must" not in needle:
            with pytest.raises(ValueError, match=needle):
                attn.attn_prefill_paged(qp, a["k_pages"], a["v_pages"], a["block_table"], a["seq_lens"])

    B, n = 2, 8
    q4 = torch.zeros(B, H, n, d, dtype=torch.bfloat16)
    k4 = torch.zeros(B, H_kv, n, d, dtype=torch.bfloat16)
    for kw, needle in ((dict(k=k4.float()), "k must be torch.bfloat16"),
                       (dict(v=k4[:, :, :4].clone()), "v must have shape"),
                       (dict(key_mask=torch.ones(B, n, dtype=torch.bool)), "key_mask must be torch.uint8"),
                       (dict(key_mask=torch.ones(B, n + 1, dtype=torch.uint8)), "key_mask must have shape"),
                       (dict(), "must be a CUDA tensor")):
        a = dict(q=q4, k=k4, v=k4.clone(), key_mask=None)
        a.update(kw)
        with pytest.raises(ValueError, match=needle):
            attn.attn_fwd(a["q"], a["k"], a["v"], 0.125, False, a["key_mask"])
    lse = torch.zeros(B, H, n, dtype=torch.float32)
    for kw, needle in ((dict(d_o=q4[:, :, :4].clone()), "d_o must have shape"),
                       (dict(lse=lse.double()), "lse must be torch.float32"),
                       (dict(o=q4.float()), "o must be torch.bfloat16"),
                       (dict(), "must be a CUDA tensor")):
        a = dict(q=q4, k=k4, v=k4.clone(), o=q4.clone(), d_o=q4.clone(), lse=lse)
        a.update(kw)
        with pytest.raises(ValueError, match=needle):
            attn.attn_bwd(a["q"], a["k"], a["v"], a["o"], a["d_o"], a["lse"], 0.125)
    q8 = torch.zeros(B, H, n, 128, dtype=torch.uint8)
    sq, sk = torch.ones(B, H, 1), torch.ones(B, H_kv, 1)
    with pytest.raises(ValueError, match="k8 must be torch.uint8"):
        attn.attn_fwd_fp8(q8, q8[:, :H_kv].to(torch.int8), q8[:, :H_kv].clone(), sq, sk, sk)
    with pytest.raises(ValueError, match="v_descale must have shape"):
        attn.attn_fwd_fp8(q8, q8[:, :H_kv].clone(), q8[:, :H_kv].clone(), sq, sk, torch.ones(B, H_kv, 2))
    with pytest.raises(ValueError, match="q_descale must be torch.float32"):
        attn.attn_fwd_fp8(q8, q8[:, :H_kv].clone(), q8[:, :H_kv].clone(), sq.double(), sk, sk)
    with pytest.raises(ValueError, match="must be a CUDA tensor"):
        attn.attn_fwd_fp8(q8, q8[:, :H_kv].clone(), q8[:, :H_kv].clone(), sq, sk, sk)
