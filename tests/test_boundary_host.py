"""The C-ABI library without a GPU: it loads, exports every function the
header declares, and rejects bad arguments before touching the device.

Only host-side code paths are exercised here (argument checks, planning,
workspace sizing, status strings); no call in this file launches a kernel.
"""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER_DIR = os.path.join(ROOT, "include")


@pytest.fixture(scope="module")
def lib():
    from transformer_attention_causal_b200 import _lib
    from transformer_attention_causal_b200.build import build

    build()
    return _lib.load()


def declared_functions():
    names = []
    for fname in os.listdir(HEADER_DIR):
        if fname.endswith(".h"):
            text = open(os.path.join(HEADER_DIR, fname)).read()
            names += re.findall(r"ATTN_API\s+[\w\s\*]+?\b(attn_\w+)\s*\(", text)
    return sorted(set(names))


def test_header_declares_the_abi():
    names = declared_functions()
    for required in ("attn_prefill", "attn_cached", "attn_cached_workspace_size",
                     "attn_status_string"):
        assert required in names


def test_library_exports_every_declared_symbol(lib):
    from transformer_attention_causal_b200 import _lib

    for name in declared_functions():
        assert hasattr(lib, name), f"{name} declared in include/ but not exported"
    out = subprocess.run(["nm", "-D", "--defined-only", _lib.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    assert set(declared_functions()) <= exported
    # nothing but the ABI is exported from the library's own code
    assert {n for n in exported if n.startswith("attn_")} == set(declared_functions())


def test_status_strings_and_version(lib):
    from transformer_attention_causal_b200 import _lib

    for code in range(7):
        assert isinstance(_lib.status_string(code), str) and _lib.status_string(code)
    assert _lib.status_string(99) == "unknown status"
    assert lib.attn_version() >= 100


F32, BF16, F16 = 0, 1, 2
FAKE = ctypes.c_void_p(0x10000)      # 16-byte aligned, never dereferenced
MISALIGNED = ctypes.c_void_p(0x10008)


def prefill(lib, q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=None, dt=BF16, B=1, H=4, Hkv=2, T=8, d=64,
            scale=0.125, causal=1):
    return lib.attn_prefill(q, k, v, o, lse, dt, B, H, Hkv, T, d, scale, causal, None)


def cached(lib, q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=None, dt=BF16, B=1, H=4, Hkv=2, Tnew=1, S=8,
           S_cap=8, d=64, start_pos=7, scale=0.125, ws=None, ws_bytes=0):
    return lib.attn_cached(q, k, v, o, lse, dt, B, H, Hkv, Tnew, S, S_cap, d, start_pos, scale, ws,
                           ws_bytes, None)


INVALID, UNSUPPORTED, WORKSPACE = 1, 2, 3


@pytest.mark.parametrize("kwargs", [
    dict(q=None), dict(k=None), dict(v=None), dict(o=None),
    dict(q=MISALIGNED), dict(o=MISALIGNED), dict(lse=ctypes.c_void_p(0x10002)),
    dict(B=-1), dict(H=-2), dict(T=-1), dict(d=-8), dict(d=0),
    dict(Hkv=0), dict(H=6, Hkv=4), dict(dt=7),
    dict(scale=float("nan")), dict(scale=float("inf")),
])
def test_prefill_rejects_invalid_arguments(lib, kwargs):
    assert prefill(lib, **kwargs) == INVALID


def test_prefill_rejects_oversized_head(lib):
    assert prefill(lib, d=264) == UNSUPPORTED


@pytest.mark.parametrize("kwargs", [
    dict(start_pos=8),                 # start_pos + Tnew > S
    dict(S=9, S_cap=8, start_pos=8),   # S > S_cap
    dict(start_pos=-1),
    dict(Tnew=3, start_pos=6),         # 6 + 3 > 8
    dict(q=None), dict(k=MISALIGNED),
])
def test_cached_rejects_invalid_arguments(lib, kwargs):
    assert cached(lib, **kwargs) == INVALID


def test_cached_reports_a_short_workspace(lib):
    need = lib.attn_cached_workspace_size(BF16, 64, 32, 8, 1, 8192, 128, 8191)
    assert need > 0
    args = dict(B=64, H=32, Hkv=8, Tnew=1, S=8192, S_cap=8192, d=128, start_pos=8191)
    assert cached(lib, ws=None, ws_bytes=0, **args) == WORKSPACE
    assert cached(lib, ws=FAKE, ws_bytes=need - 1, **args) == WORKSPACE
    assert cached(lib, ws=MISALIGNED, ws_bytes=need, **args) == INVALID


def test_chunked_prefill_pieces_need_their_workspace(lib):
    """A chunked prefill whose last pass is cut into pieces needs the
    workspace attn_cached_workspace_size reports; less is rejected before
    anything is launched (host only: the pointers are never dereferenced)."""
    F16 = 2
    args = dict(dt=F16, B=32, H=8, Hkv=1, Tnew=512, S=4096, S_cap=4096, d=128, start_pos=3584)
    need = lib.attn_cached_workspace_size(F16, 32, 8, 1, 512, 4096, 128, 3584)
    assert need > 0
    assert cached(lib, ws=None, ws_bytes=0, **args) == WORKSPACE
    assert cached(lib, ws=FAKE, ws_bytes=need - 1, **args) == WORKSPACE
    assert cached(lib, ws=MISALIGNED, ws_bytes=need, **args) == INVALID
    # the paged form, planned at its length bound
    need_p = lib.attn_cached_paged_workspace_size(F16, 32, 8, 1, 512, 128, 4096)
    assert need_p == need
    pargs = dict(dt=F16, B=32, H=8, Hkv=1, Tnew=512, d=128, max_pages=32, num_pages=1024,
                 page_size=128, max_kv_len=4096)
    assert paged(lib, ws=None, ws_bytes=0, **pargs) == WORKSPACE
    assert paged(lib, ws=FAKE, ws_bytes=need_p - 1, **pargs) == WORKSPACE


def test_empty_problems_are_a_no_op(lib):
    # B * H * Tq == 0: nothing is launched, null pointers allowed
    assert prefill(lib, q=None, k=None, v=None, o=None, B=0) == 0
    assert prefill(lib, q=None, k=None, v=None, o=None, T=0) == 0
    assert cached(lib, q=None, k=None, v=None, o=None, Tnew=0, start_pos=8) == 0
    assert lib.attn_prefill_plan(BF16, 0, 4, 2, 8, 64, 1) == 0


def test_plans_pick_the_intended_kernels(lib):
    from transformer_attention_causal_b200 import _lib as L

    # float32 always runs on CUDA cores
    assert lib.attn_prefill_plan(F32, 1, 2, 1, 16, 8, 1) == L.KERNEL_SIMT
    # the four 16-bit workloads
    assert lib.attn_prefill_plan(BF16, 1, 32, 32, 2048, 80, 1) == L.KERNEL_TCGEN05
    assert lib.attn_prefill_plan(BF16, 8, 16, 8, 4096, 128, 1) == L.KERNEL_TCGEN05
    assert lib.attn_cached_plan(BF16, 64, 32, 8, 1, 8192, 8192, 128, 8191) == L.KERNEL_SPLITKV
    # decode at every tensor-core head size (BitNet-3B: MHA, d = 80)
    for d in (64, 80, 96, 112):
        assert lib.attn_cached_plan(BF16, 1, 32, 32, 1, 2048, 2048, d, 2047) == L.KERNEL_SPLITKV
    assert lib.attn_cached_plan(BF16, 1, 32, 32, 17, 2048, 2048, 80, 2031) == L.KERNEL_TCGEN05
    # head sizes off the tensor-core grid decode on CUDA cores; d = 256 takes
    # the CUDA-core split-KV kernel up to 8 rows per K/V head
    for d in (48, 72, 136, 192):
        assert lib.attn_cached_plan(BF16, 1, 32, 32, 1, 2048, 2048, d, 2047) == L.KERNEL_SIMT
    assert lib.attn_cached_plan(BF16, 1, 32, 32, 1, 2048, 2048, 256, 2047) == L.KERNEL_SPLITKV
    assert lib.attn_cached_plan(BF16, 1, 32, 8, 5, 2048, 2048, 256, 2043) == L.KERNEL_SIMT
    assert lib.attn_cached_plan(F16, 32, 8, 1, 512, 4096, 4096, 128, 3584) == L.KERNEL_TCGEN05
    # head sizes the tensor-core kernel does not take fall back to CUDA cores
    assert lib.attn_prefill_plan(BF16, 1, 2, 1, 16, 40, 1) == L.KERNEL_SIMT
    assert lib.attn_prefill_plan(BF16, 1, 2, 1, 16, 200, 1) == L.KERNEL_SIMT
    # rejected arguments
    assert lib.attn_prefill_plan(BF16, 1, 3, 2, 16, 64, 1) == -1


def test_chunked_prefill_tail_pieces_workspace(lib):
    """The tensor-core chunked prefill cuts the units of its last pass into
    pieces of their key range when that pass would leave most of the 148 SMs
    idle; the workspace holds each piece's fp32 O rows and one log2-sum-exp
    per row."""
    F16 = 2
    # MQA chunked prefill (B=32, H=8/1, 512 new tokens at 3584 over 4096
    # keys, d=128): 512 units, 3 full passes, 68 units left, 2 pieces each
    assert lib.attn_cached_workspace_size(F16, 32, 8, 1, 512, 4096, 128, 3584) == 68 * 2 * 2 * 128 * 129 * 4
    # a single unit (B=1, H=2/1, 64 new tokens over 4064 keys, d=112): 4 pieces
    assert lib.attn_cached_workspace_size(BF16, 1, 2, 1, 64, 4064, 112, 4000) == 4 * 2 * 128 * 113 * 4
    # 2048 units (13 full passes, 124 left of 148): not cut
    assert lib.attn_cached_workspace_size(BF16, 8, 16, 8, 4096, 4096, 128, 0) == 0
    # a short history: no piece would keep 4 key tiles
    assert lib.attn_cached_workspace_size(F16, 2, 8, 1, 200, 500, 128, 300) == 0
    # a local window is never cut
    assert lib.attn_cached_local_workspace_size(F16, 32, 8, 1, 512, 4096, 128, 3584, 1024) == 0
    # the paged form plans with the length bound
    assert lib.attn_cached_paged_workspace_size(F16, 32, 8, 1, 512, 128, 4096) == 68 * 2 * 2 * 128 * 129 * 4


def test_workspace_size_is_zero_without_splits(lib):
    # a single long sequence on one K/V head still splits; a tiny history does not
    assert lib.attn_cached_workspace_size(BF16, 1, 4, 4, 1, 64, 128, 63) == 0
    assert lib.attn_cached_workspace_size(BF16, 1, 4, 1, 1, 65536, 128, 65535) > 0
    # rejected arguments report 0
    assert lib.attn_cached_workspace_size(BF16, 1, 4, 3, 1, 64, 128, 63) == 0


def test_split_counts_of_the_decode_planner(lib):
    """The split count, read back from the workspace size (fp32 partials:
    units x splits x rows x (d + 2) floats, rounded up to 256 bytes).  The
    planner models a call as waves of CTAs over 148 SMs, each CTA costing
    its 128-key stages plus about three stages of start-up and merge."""
    def splits(B, H, Hkv, S, d):
        ws = lib.attn_cached_workspace_size(BF16, B, H, Hkv, 1, S, d, S - 1)
        per_split = B * Hkv * (H // Hkv) * (d + 2) * 4
        n = ws // per_split
        assert ws == 0 or (ws - n * per_split) < 256
        return max(n, 1)
    # GQA decode, 512 units of 64 stages: 2 splits (7 waves of 32-stage CTAs)
    assert splits(64, 32, 8, 8192, 128) == 2
    # 64 units: one wave of 128 CTAs beats 7 waves of 4-stage CTAs
    assert splits(8, 32, 8, 8192, 128) == 2
    # MHA d = 80, 256 units of 32 stages: no split (two waves)
    assert splits(8, 32, 32, 4096, 80) == 1
    # one sequence on one K/V head, 157 stages: 79 splits of 2 (one wave)
    assert splits(1, 4, 1, 20000, 128) == 79


def append(lib, k=FAKE, v=FAKE, kc=FAKE, vc=FAKE, dt=BF16, B=1, Hkv=2, Tnew=4, S_cap=16, d=64,
           start_pos=3, base=10000.0):
    return lib.attn_kv_append_rope(k, v, kc, vc, dt, B, Hkv, Tnew, S_cap, d, start_pos, base, None)


@pytest.mark.parametrize("kwargs", [
    dict(k=None), dict(v=None), dict(kc=None), dict(vc=None),
    dict(kc=MISALIGNED), dict(v=MISALIGNED),
    dict(start_pos=13),                # 13 + 4 > 16
    dict(start_pos=-1), dict(B=-1), dict(Tnew=-2), dict(S_cap=-1),
    dict(d=0), dict(d=60), dict(d=6, dt=F32), dict(dt=5),
    dict(base=float("nan")), dict(base=float("inf")),
])
def test_append_rejects_invalid_arguments(lib, kwargs):
    assert append(lib, **kwargs) == INVALID


def test_append_limits_and_empty_calls(lib):
    assert append(lib, d=264) == UNSUPPORTED
    assert append(lib, d=260, dt=F32) == UNSUPPORTED
    # nothing to write: no launch, null pointers allowed
    assert append(lib, k=None, v=None, kc=None, vc=None, Tnew=0) == 0
    assert append(lib, k=None, v=None, kc=None, vc=None, B=0) == 0


def paged(lib, q=FAKE, kp=FAKE, vp=FAKE, o=FAKE, dt=BF16, B=2, H=8, Hkv=2, Tnew=1, d=128,
          table=ctypes.c_void_p(0x20000), max_pages=4, num_pages=8, page_size=16,
          lens=ctypes.c_void_p(0x30000), max_kv_len=64, scale=0.1, ws=None, ws_bytes=0):
    return lib.attn_cached_paged(q, kp, vp, o, None, dt, B, H, Hkv, Tnew, d, table, max_pages,
                                 num_pages, page_size, lens, max_kv_len, scale, ws, ws_bytes, None)


@pytest.mark.parametrize("kwargs", [
    dict(table=None), dict(lens=None), dict(table=ctypes.c_void_p(0x20002)),
    dict(page_size=12), dict(page_size=4), dict(page_size=0),
    dict(max_kv_len=65),                 # > max_pages * page_size
    dict(max_kv_len=0, Tnew=1),          # < Tnew
    dict(num_pages=0), dict(q=None), dict(kp=MISALIGNED), dict(scale=float("nan")),
    dict(H=6, Hkv=4), dict(dt=7),
])
def test_paged_rejects_invalid_arguments(lib, kwargs):
    assert paged(lib, **kwargs) == INVALID


def test_paged_limits(lib):
    assert paged(lib, dt=F32) == UNSUPPORTED            # float32 has no paged kernel
    # many rows per K/V head go to the tensor-core prefill, which takes d in
    # [64, 128]; other head sizes have no paged kernel
    assert paged(lib, H=32, Hkv=1, Tnew=1, d=48) == UNSUPPORTED
    assert paged(lib, H=32, Hkv=1, Tnew=1, d=256) == UNSUPPORTED
    assert paged(lib, d=72) == UNSUPPORTED
    # empty problems launch nothing
    assert paged(lib, q=None, kp=None, vp=None, o=None, table=None, lens=None, B=0) == 0
    # a split plan needs workspace
    need = lib.attn_cached_paged_workspace_size(BF16, 64, 32, 8, 1, 128, 8192)
    assert need > 0
    assert paged(lib, B=64, H=32, Hkv=8, max_pages=128, num_pages=8192, page_size=64,
                 max_kv_len=8192) == WORKSPACE
    assert lib.attn_cached_paged_workspace_size(F32, 64, 32, 8, 1, 128, 8192) == 0


def backward(lib, q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=FAKE, do=FAKE, dq=FAKE, dk=FAKE, dv=FAKE,
             dt=BF16, B=1, H=4, Hkv=2, T=300, d=128, scale=0.125, causal=1, ws=FAKE,
             ws_bytes=1 << 20):
    return lib.attn_prefill_backward(q, k, v, o, lse, do, dq, dk, dv, dt, B, H, Hkv, T, d, scale,
                                     causal, ws, ws_bytes, None)


@pytest.mark.parametrize("kwargs", [
    dict(q=None), dict(k=None), dict(v=None), dict(o=None), dict(lse=None), dict(do=None),
    dict(dq=None), dict(dk=None), dict(dv=None), dict(dq=MISALIGNED), dict(do=MISALIGNED),
    dict(lse=ctypes.c_void_p(0x10002)), dict(ws=MISALIGNED),
    dict(B=-1), dict(T=-1), dict(Hkv=0), dict(H=6, Hkv=4), dict(dt=7), dict(scale=float("nan")),
])
def test_backward_rejects_invalid_arguments(lib, kwargs):
    assert backward(lib, **kwargs) == INVALID


def test_backward_rejects_unsupported_shapes(lib):
    # float32 and 16-bit head sizes off the tensor-core set run on CUDA cores;
    # only d > 256 is refused
    assert backward(lib, d=264) == UNSUPPORTED
    for kwargs in (dict(dt=F32), dict(d=48), dict(d=136), dict(d=72), dict(dt=F32, d=256)):
        assert backward(lib, ws=None, ws_bytes=0, **kwargs) == WORKSPACE


def test_backward_local_rejects_a_negative_window(lib):
    assert lib.attn_prefill_backward_local(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, BF16, 1,
                                           4, 2, 300, 128, 0.125, -1, FAKE, 1 << 20, None) == INVALID


def test_backward_workspace(lib):
    # two float32 row statistics per padded query row: 300 rows pad to 384
    need = lib.attn_prefill_backward_workspace_size(BF16, 2, 4, 2, 300, 128)
    assert need == 2 * 2 * 4 * 384 * 4
    assert lib.attn_prefill_backward_workspace_size(F32, 2, 4, 2, 300, 128) == need
    assert lib.attn_prefill_backward_workspace_size(BF16, 2, 4, 2, 0, 128) == 0
    assert backward(lib, B=2, ws=FAKE, ws_bytes=need - 1) == WORKSPACE
    assert backward(lib, B=2, ws=None, ws_bytes=need) == WORKSPACE


def test_backward_empty_problem(lib):
    # T = 0: nothing to do, null pointers allowed
    assert backward(lib, q=None, k=None, v=None, o=None, lse=None, do=None, dq=None, dk=None,
                    dv=None, ws=None, ws_bytes=0, T=0) == 0
