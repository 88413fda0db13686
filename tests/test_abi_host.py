"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every entry point include/kda.h declares, sizes workspaces, and rejects bad
arguments synchronously (before any CUDA call)."""
import ctypes
import os
import re

import pytest

from gated_delta_rule_98_b200 import kda

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    from gated_delta_rule_98_b200 import build
    build.build()
    return kda.lib()


def declared_entry_points():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names |= set(re.findall(r"\b(kda_[a-z0-9_]+)\s*\(", src))
    return names


def test_exports_every_declared_symbol(L):
    declared = declared_entry_points()
    assert declared >= {"kda_forward", "kda_decode_step", "kda_forward_workspace_size"}
    for name in declared:
        assert hasattr(L, name), f"libkda.so does not export {name}"
    assert set(kda.EXPORTS) == declared


def test_status_strings(L):
    for s, name in [(0, "KDA_OK"), (-1, "KDA_ERR_INVALID_ARG"), (-2, "KDA_ERR_UNSUPPORTED"),
                    (-3, "KDA_ERR_CUDA"), (-4, "KDA_ERR_TIMEOUT")]:
        assert kda.status_string(s) == name
    assert L.kda_version() >= 100


def test_workspace_size(L):
    ws = kda.kda_forward_workspace_size
    assert ws(1, 4096, 4096, 16, 128, 128, kda.KDA_BF16, 64) > 0
    assert ws(1, 4096, 4096, 16, 128, 128, kda.KDA_BF16, 64) >= \
        ws(1, 2048, 2048, 16, 128, 128, kda.KDA_BF16, 64)
    assert ws(1, 64, 64, 2, 48, 32, kda.KDA_F32, 16) == 0       # unsupported dk
    assert ws(1, 64, 64, 2, 32, 32, kda.KDA_F32, 32) == 0       # unsupported chunk
    assert ws(1, 64, 64, 2, 32, 32, 7, 16) == 0                 # unsupported dtype
    assert ws(-1, 64, 64, 2, 32, 32, kda.KDA_F32, 16) == 0
    assert ws(0, 0, 0, 2, 32, 32, kda.KDA_F32, 16) > 0          # empty problem: header only


def test_workspace_holds_one_chunk_slot_per_chunk_and_head(L):
    """The bf16 tensor-core path stores one chunk slot of 74,496 bytes per
    (chunk, head) for every chunk id cu[n]/64 + n + j below T/64 + N, whether
    the sequences are cut into segments (one long sequence, few heads) or not
    (many sequences x heads); the segment maps add at most a few MB."""
    ws = kda.kda_forward_workspace_size
    slot = 74496
    for N, T, H in ((1, 4096, 16), (1, 65536, 16), (1, 8192, 4), (8, 8 * 4096, 16)):
        size = ws(N, T, T // N, H, 128, 128, kda.KDA_BF16, 64)
        need = (T // 64 + N) * H * slot
        assert need <= size <= need + 64 * 1024 * 1024, (N, T, H, size, need)


@pytest.mark.parametrize("N,H,L,P", [
    (1, 16, 65536, 9),    # 148 // 16
    (1, 4, 4096, 16),     # 148 // 4 = 37, at most 16
    (1, 16, 256, 2),      # 4 chunks: at most half the chunk count
    (1, 16, 64, 1),       # one chunk
    (8, 16, 4096, 1),     # 128 (sequence, head) pairs fill the SMs without segments
    (2, 32, 4096, 2),     # 64 pairs: 148 // 64
    (1, 200, 4096, 1),
])
def test_segment_rule(L, N, H, P):
    """Segments per sequence on the tensor-core path, P = 148 // (N H), at most
    half the chunk count and at most 16 (1 when the pairs fill the SMs): the
    workspace holds (3P - 2) 64 KB state maps per (sequence, head) before the
    chunk slots, and the call makes 4 launches when P > 1, else 2."""
    T = N * L
    size = kda.kda_forward_workspace_size(N, T, L, H, 128, 128, kda.KDA_BF16, 64)
    maps = size - (T // 64 + N) * H * 74496 - 256           # header, then the maps
    assert maps >= 0 and maps // (N * H * 65536) == 3 * P - 2, (size, maps)
    assert kda.kda_forward_launches(N, T, L, H, 128, 128, kda.KDA_BF16, 64) == (4 if P > 1 else 2)
    # context parallelism keeps room for all P transitions (P + 1 segment buffers)
    cw = kda.kda_cp_workspace_size(N, T, L, H, 128, 128, kda.KDA_BF16, 64)
    cmaps = cw - (T // 64 + N) * H * 74496 - 256
    assert cmaps // (N * H * 65536) == 3 * (P + 1) - 2


FAKE = 0x10000  # aligned fake device address: never dereferenced by these calls


def _fwd(**over):
    a = dict(q=FAKE, k=FAKE, v=FAKE, z=FAKE, A=FAKE, beta=FAKE, S0=None, cu=None, N=1, T=64,
             L=64, H=2, dk=32, dv=32, dt=kda.KDA_F32, chunk=16, o=FAKE, Sf=FAKE, ws=FAKE,
             wsb=1 << 40, stream=None)
    a.update(over)
    return kda.kda_forward(a["q"], a["k"], a["v"], a["z"], a["A"], a["beta"], a["S0"], a["cu"],
                           a["N"], a["T"], a["L"], a["H"], a["dk"], a["dv"], a["dt"], a["chunk"],
                           a["o"], a["Sf"], a["ws"], a["wsb"], a["stream"])


@pytest.mark.parametrize("over,want", [
    (dict(q=None), kda.KDA_ERR_INVALID_ARG),
    (dict(z=None), kda.KDA_ERR_INVALID_ARG),
    (dict(A=None), kda.KDA_ERR_INVALID_ARG),
    (dict(o=None), kda.KDA_ERR_INVALID_ARG),
    (dict(ws=None), kda.KDA_ERR_INVALID_ARG),
    (dict(wsb=16), kda.KDA_ERR_INVALID_ARG),
    (dict(q=FAKE + 8), kda.KDA_ERR_INVALID_ARG),
    (dict(beta=FAKE + 2), kda.KDA_ERR_INVALID_ARG),
    (dict(ws=FAKE + 4), kda.KDA_ERR_INVALID_ARG),
    (dict(T=65), kda.KDA_ERR_INVALID_ARG),          # T != N * max_seqlen without cu_seqlens
    (dict(H=0), kda.KDA_ERR_INVALID_ARG),
    (dict(N=-1), kda.KDA_ERR_INVALID_ARG),
    (dict(dk=48), kda.KDA_ERR_UNSUPPORTED),
    (dict(dv=256), kda.KDA_ERR_UNSUPPORTED),
    (dict(chunk=32), kda.KDA_ERR_UNSUPPORTED),
    (dict(dt=5), kda.KDA_ERR_UNSUPPORTED),
])
def test_forward_rejects_bad_arguments(L, over, want):
    assert _fwd(**over) == want


def test_forward_g_and_decode_reject_bad_arguments(L):
    st = kda.kda_forward_g(FAKE, FAKE, FAKE, None, FAKE, None, None, 1, 64, 64, 2, 32, 32,
                           kda.KDA_F32, 16, FAKE, None, FAKE, 1 << 40, None)
    assert st == kda.KDA_ERR_INVALID_ARG
    dec = kda.kda_decode_step
    assert dec(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, 4, 2, 32, 32, kda.KDA_F32, FAKE,
               None) == kda.KDA_ERR_INVALID_ARG
    assert dec(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 4, 2, 96, 32, kda.KDA_F32, FAKE,
               None) == kda.KDA_ERR_UNSUPPORTED
    assert dec(FAKE + 4, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 4, 2, 32, 32, kda.KDA_F32, FAKE,
               None) == kda.KDA_ERR_INVALID_ARG
    # B = 0 is a no-op that touches nothing
    assert dec(None, None, None, None, None, None, None, 0, 2, 32, 32, kda.KDA_F32, None,
               None) == kda.KDA_OK
    assert kda.kda_check_device_error(None, None) == kda.KDA_ERR_INVALID_ARG


def test_binding_rejects_cpu_tensors(L):
    import torch
    q = torch.zeros(4, 1, 32)
    with pytest.raises(ValueError):
        kda.decode_step(q, q, q, q, torch.zeros(1), torch.zeros(4, 1), torch.zeros(4, 1, 32, 32))


def test_checkpoints_reject_bad_interval_and_buffer(L):
    def ck(**over):
        a = dict(interval=64, S_ckpt=FAKE, chunk=16)
        a.update(over)
        return kda.kda_forward_checkpoints(
            FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, None, 1, 128, 128, 2, 32, 32,
            kda.KDA_F32, a["chunk"], FAKE, FAKE, a["S_ckpt"], a["interval"], FAKE, 1 << 40, None)
    assert ck(interval=0) == kda.KDA_ERR_INVALID_ARG
    assert ck(interval=-16) == kda.KDA_ERR_INVALID_ARG
    assert ck(interval=24) == kda.KDA_ERR_INVALID_ARG          # not a multiple of the chunk
    assert ck(S_ckpt=None) == kda.KDA_ERR_INVALID_ARG          # 2 checkpoints need a buffer
    assert ck(S_ckpt=FAKE + 4) == kda.KDA_ERR_INVALID_ARG      # misaligned
    assert ck(chunk=32) == kda.KDA_ERR_UNSUPPORTED


def test_norm_gate_rejects_bad_epilogue_arguments(L):
    def fw(gate=FAKE, w=None, eps=1e-6, T=128):
        return kda.kda_forward_norm_gate(
            FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, None, 1, T, T, 2, 32, 32,
            kda.KDA_F32, 16, gate, w, eps, FAKE, FAKE, FAKE, 1 << 40, None)
    assert fw(gate=None) == kda.KDA_ERR_INVALID_ARG             # gate input required
    assert fw(gate=FAKE + 8) == kda.KDA_ERR_INVALID_ARG         # misaligned
    assert fw(w=FAKE + 4) == kda.KDA_ERR_INVALID_ARG
    assert fw(eps=-1e-6) == kda.KDA_ERR_INVALID_ARG
    assert fw(eps=float("nan")) == kda.KDA_ERR_INVALID_ARG
    assert fw(eps=float("inf")) == kda.KDA_ERR_INVALID_ARG

    def dec(gate=FAKE, eps=1e-6, B=4, dk=32):
        return kda.kda_decode_step_norm_gate(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, B, 2, dk,
                                             32, kda.KDA_F32, gate, None, eps, FAKE, None)
    assert dec(gate=None) == kda.KDA_ERR_INVALID_ARG
    assert dec(eps=float("nan")) == kda.KDA_ERR_INVALID_ARG
    assert dec(dk=48) == kda.KDA_ERR_UNSUPPORTED
    assert dec(gate=None, B=0) == kda.KDA_OK                    # nothing to do


def test_decode_conv_rejects_bad_arguments(L):
    def dec(width=4, wq=FAKE, state=FAKE, B=4, dk=32):
        return kda.kda_decode_step_conv(FAKE, FAKE, FAKE, wq, FAKE, FAKE, width, state, FAKE,
                                        FAKE, FAKE, FAKE, B, 2, dk, 32, kda.KDA_F32, FAKE, None)
    assert dec(width=0) == kda.KDA_ERR_UNSUPPORTED
    assert dec(width=5) == kda.KDA_ERR_UNSUPPORTED
    assert dec(wq=None) == kda.KDA_ERR_INVALID_ARG
    assert dec(wq=FAKE + 2) == kda.KDA_ERR_INVALID_ARG          # taps are 4-byte aligned
    assert dec(state=None) == kda.KDA_ERR_INVALID_ARG           # width 4 carries a window
    assert dec(state=FAKE + 2) == kda.KDA_ERR_INVALID_ARG       # fp32 window, misaligned
    assert dec(dk=48) == kda.KDA_ERR_UNSUPPORTED
    assert dec(state=None, wq=None, B=0) == kda.KDA_OK          # nothing to do


def test_scalar_gate_requires_the_gate(L):
    st = kda.kda_forward_scalar_gate(FAKE, FAKE, FAKE, None, FAKE, None, None, 1, 64, 64, 2, 32,
                                     32, kda.KDA_F32, 16, FAKE, FAKE, FAKE, 1 << 40, None)
    assert st == kda.KDA_ERR_INVALID_ARG
    st = kda.kda_forward_scalar_gate(FAKE, FAKE, FAKE, FAKE + 4, FAKE, None, None, 1, 64, 64, 2,
                                     32, 32, kda.KDA_F32, 16, FAKE, FAKE, FAKE, 1 << 40, None)
    assert st == kda.KDA_ERR_INVALID_ARG


def test_short_conv_swish_rejects_bad_arguments(L):
    def sc(x=FAKE, w=FAKE, channels=64, width=4, T=32, N=1, Lm=32):
        return kda.kda_short_conv_swish(x, w, None, N, T, Lm, channels, width, kda.KDA_BF16, FAKE,
                                        None)
    assert sc(width=0) == kda.KDA_ERR_UNSUPPORTED
    assert sc(width=5) == kda.KDA_ERR_UNSUPPORTED
    assert sc(channels=12) == kda.KDA_ERR_UNSUPPORTED
    assert sc(x=FAKE + 8) == kda.KDA_ERR_INVALID_ARG
    assert sc(w=None) == kda.KDA_ERR_INVALID_ARG
    assert sc(T=33) == kda.KDA_ERR_INVALID_ARG                  # N * max_seqlen != T
    assert sc(T=0, Lm=0) == kda.KDA_OK


def test_forward_conv_workspace_and_arguments(L):
    args = (2, 256, 128, 4, 128, 128, kda.KDA_BF16, 64)
    fw = kda.kda_forward_workspace_size(*args)
    cw = kda.kda_forward_conv_workspace_size(*args)
    # tensor-core path: the prologue runs inside the chunk preparation
    assert cw == fw > 0
    # CUDA-core path: the prologue's q, k, v (fp32) follow the forward's workspace
    args32 = (2, 256, 128, 4, 64, 64, kda.KDA_F32, 16)
    fw32 = kda.kda_forward_workspace_size(*args32)
    assert kda.kda_forward_conv_workspace_size(*args32) >= fw32 + 3 * 256 * 4 * 64 * 4
    assert kda.kda_forward_conv_workspace_size(2, 256, 128, 4, 48, 128, kda.KDA_BF16, 64) == 0

    def fc(ws_bytes=cw, width=4, wq=FAKE):
        return kda.kda_forward_conv(FAKE, FAKE, FAKE, wq, FAKE, FAKE, width, FAKE, FAKE, FAKE,
                                    None, None, 2, 256, 128, 4, 128, 128, kda.KDA_BF16, 64, FAKE,
                                    FAKE, FAKE, ws_bytes, None)
    assert fc(ws_bytes=cw - 1) == kda.KDA_ERR_INVALID_ARG
    assert fc(width=0) == kda.KDA_ERR_UNSUPPORTED
    assert fc(wq=None) == kda.KDA_ERR_INVALID_ARG


def test_binding_rejects_mismatched_shapes_before_any_launch():
    """The binding checks every tensor's shape and dtype against its role (the
    C ABI only sees pointers); the checks run before the CUDA check would."""
    import torch
    from gated_delta_rule_98_b200.kda import _shapes
    T, H, dk, dv, N = 10, 2, 32, 32, 3
    ok = dict(q=torch.empty(T, H, dk), v=torch.empty(T, H, dv), beta=torch.empty(T, H),
              S0=torch.empty(N, H, dk, dv), cu_seqlens=torch.zeros(N + 1, dtype=torch.int32))
    _shapes(T, H, dk, dv, N, torch.float32, **ok)
    bad = [dict(S0=torch.empty(1, H, dk, dv)),                  # one state for three sequences
           dict(beta=torch.empty(T, H, 1)),
           dict(cu_seqlens=torch.zeros(N + 1, dtype=torch.int64)),
           dict(A=torch.empty(H, dtype=torch.float64)),
           dict(k=torch.empty(T, H, dk, dtype=torch.bfloat16)),
           dict(out_gate=torch.empty(T, H, dk + 1)),
           dict(S_ckpt=torch.empty(N, H, 2, dk, dv + 1))]
    for b in bad:
        with pytest.raises(ValueError):
            _shapes(T, H, dk, dv, N, torch.float32, **b)


def test_cp_entry_points_reject_bad_arguments(L):
    args = (1, 512, 512, 4, 128, 128, kda.KDA_BF16, 64)
    cw = kda.kda_cp_workspace_size(*args)
    assert cw > kda.kda_forward_workspace_size(*args)
    assert kda.kda_cp_workspace_size(1, 512, 512, 4, 64, 64, kda.KDA_BF16, 64) == 0
    assert kda.kda_cp_workspace_size(1, 512, 512, 4, 128, 128, kda.KDA_F32, 64) == 0

    def loc(ws_bytes=cw, M=FAKE, dt=kda.KDA_BF16):
        return kda.kda_cp_local(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, 1, 512, 512, 4, 128,
                                128, dt, 64, M, FAKE, FAKE, ws_bytes, None)
    assert loc(ws_bytes=cw - 1) == kda.KDA_ERR_INVALID_ARG
    assert loc(M=None) == kda.KDA_ERR_INVALID_ARG
    assert loc(dt=kda.KDA_F32) == kda.KDA_ERR_UNSUPPORTED

    def fin(ws_bytes=cw, o=FAKE):
        return kda.kda_cp_finish(None, None, 1, 512, 512, 4, 128, 128, kda.KDA_BF16, 64, o, None,
                                 FAKE, ws_bytes, None)
    assert fin(ws_bytes=cw - 1) == kda.KDA_ERR_INVALID_ARG
    assert fin(o=None) == kda.KDA_ERR_INVALID_ARG
    assert kda.kda_state_compose(FAKE, FAKE, None, FAKE, 2, 128, 48, None) == \
        kda.KDA_ERR_UNSUPPORTED
    assert kda.kda_state_compose(FAKE, None, None, FAKE, 2, 128, 128, None) == \
        kda.KDA_ERR_INVALID_ARG
    assert kda.kda_state_compose(None, None, None, None, 0, 128, 128, None) == kda.KDA_OK


def test_empty_problem_sizes_on_the_tensor_core_path(L):
    """num_seqs = 0 on the bf16 d=128 chunk-64 path: the sizing calls return
    the header-only workspace and no launches instead of failing."""
    bf = kda.KDA_BF16
    assert kda.kda_forward_workspace_size(0, 0, 0, 16, 128, 128, bf, 64) > 0
    assert kda.kda_forward_launches(0, 0, 0, 16, 128, 128, bf, 64) == 0
    assert kda.kda_forward_conv_workspace_size(0, 0, 0, 16, 128, 128, bf, 64) > 0
    assert kda.kda_cp_workspace_size(0, 0, 0, 16, 128, 128, bf, 64) > 0
    # (sequence, head) counts whose product overflows 32 bits still size
    assert kda.kda_forward_workspace_size(70000, 70000, 1, 70000, 128, 128, bf, 64) > 0
