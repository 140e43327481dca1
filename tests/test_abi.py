"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every function include/gdn.h declares, sizes workspaces, and rejects bad
arguments before any launch."""
import ctypes
import os
import re

import pytest

from gated_delta_rule_81_b200 import build, gdn

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return gdn.load()


def declared_functions():
    text = open(os.path.join(ROOT, "include", "gdn.h")).read()
    return sorted(set(re.findall(r"^\s*(?:size_t|gdn_status|const char\*|long long|int)\s+(gdn_\w+)\s*\(", text, re.M)))


def test_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert set(names) >= set(gdn.EXPORTS)
    for n in names:
        assert hasattr(lib, n), n


def test_debug_library_exports_the_same_symbols(lib):
    """libgdn_debug.so (bounds-checked workspace accesses) is a drop-in for libgdn.so."""
    dbg = gdn.load(build.lib_path("libgdn_debug.so"), fresh=True)
    assert dbg is not lib
    for n in declared_functions():
        assert hasattr(dbg, n), n


def test_status_strings(lib):
    for code in range(8):
        assert gdn.status_string(code).startswith("GDN_")


def test_workspace_size(lib):
    base = gdn.workspace_size(16, 48, 1, 0)
    assert base > 0
    per_chunk = gdn.workspace_size(16, 48, 1, 1) - base
    assert per_chunk == 16 * 32768 + 48 * 132096  # K image per key head; W, gamma Q, P, B_U, v_hat, gates per value head
    assert gdn.workspace_size(0, 48, 1, 1) == 0
    assert gdn.workspace_size(16, 48, -1, 1) == 0


def fake_inputs(H_k=2, H_v=6, ptr=0x10000):
    s = gdn.GdnInputs()
    for f in ("q", "k", "v", "a", "b", "z", "conv_w", "A_log", "norm_w"):
        setattr(s, f, ptr)
    s.stride_q = s.stride_k = H_k * 128
    s.stride_v = s.stride_z = H_v * 128
    s.stride_a = s.stride_b = H_v
    s.H_k, s.H_v, s.scale = H_k, H_v, 1.0
    return s


def call_prefill(lib, s, B=1, T=64, out=0x900000, ws=0x2000000, ws_bytes=1 << 30, conv_in=None, conv_out=None,
                 state_in=None, state_out=None):
    return lib.gdn_prefill(ctypes.byref(s), B, T, state_in, state_out, conv_in, conv_out, out, ws, ws_bytes, None,
                           None)


def test_rejects_bad_shapes(lib):
    s = fake_inputs(H_k=4, H_v=6)  # 6 % 4 != 0
    assert call_prefill(lib, s) == 1
    s = fake_inputs(H_k=1, H_v=16)  # group of 16 value heads per key head
    assert call_prefill(lib, s) == 2
    s = fake_inputs()
    s.stride_q = 100  # below H_k * 128
    assert call_prefill(lib, s) == 1
    assert call_prefill(lib, fake_inputs(), B=-1) == 1


def test_rejects_null_and_misaligned(lib):
    s = fake_inputs()
    s.z = None
    assert call_prefill(lib, s) == 1
    s = fake_inputs()
    s.q = 0x10008  # 8-byte aligned only
    assert call_prefill(lib, s) == 3
    s = fake_inputs()
    s.stride_v = 6 * 128 + 4  # token stride not a multiple of 16 bytes
    assert call_prefill(lib, s) == 3
    assert call_prefill(lib, fake_inputs(), out=0x900008) == 3


def test_rejects_aliasing_and_small_workspace(lib):
    s = fake_inputs()
    assert call_prefill(lib, s, conv_in=0x5000000, conv_out=0x5000000 + 16) == 4
    assert call_prefill(lib, s, out=0x10000) == 4  # out over the inputs
    assert call_prefill(lib, s, state_in=0x7000000, state_out=0x7000000 + 4096) == 4
    assert call_prefill(lib, s, state_in=0x7000000, state_out=0x7000000) != 4  # in place is allowed
    assert call_prefill(lib, s, ws_bytes=1024) == 7
    assert call_prefill(lib, s, ws=None) == 7


def test_prefill_rejects_every_written_buffer_overlap(lib):
    """One rule for every prefill entry point: a buffer the call writes (state_out, conv_out,
    out) overlaps no other state, conv or output buffer (state_out == state_in excepted), and
    none of them lies in the workspace."""
    s = fake_inputs()  # T = 64 tokens at 2 / 6 heads: out is 64 * 6 * 128 * 2 = 98,304 bytes
    out = 0x900000
    assert call_prefill(lib, s, conv_out=out + 1024) == 4                     # conv_out over out
    assert call_prefill(lib, s, state_out=out + 4096) == 4                    # state_out over out
    assert call_prefill(lib, s, conv_in=0x5000000, state_out=0x5000000) == 4  # state_out over conv_in
    assert call_prefill(lib, s, conv_out=0x5000000, state_out=0x5000000) == 4  # state_out over conv_out
    assert call_prefill(lib, s, state_in=0x5000000, conv_out=0x5000000) == 4  # conv_out over state_in
    assert call_prefill(lib, s, state_in=0x2000000 + 4096) == 4               # state_in inside the workspace
    assert call_prefill(lib, s, out=0x2000000 + 1024) == 4                    # out inside the workspace


def test_err_status_maps_device_error_bits(lib):
    assert gdn.err_status(0) == 0
    assert gdn.err_status(1) == 6 and gdn.err_status(1 | 4) == 6   # a timed-out wait wins
    for bit in (4, 8, 16, 32):
        assert gdn.err_status(bit) == 1
    assert gdn.status_string(6).startswith("GDN_ERR_DEVICE_TIMEOUT")


def test_varlen_rejects_bad_cu_seqlens(lib):
    s = fake_inputs()
    for host in ([1, 5, 9], [0, 9, 5]):
        arr = (ctypes.c_int * 3)(*host)
        rc = lib.gdn_prefill_varlen(ctypes.byref(s), 2, 0x3000000, arr, None, None, None, None, 0x900000, 0x2000000,
                                    1 << 30, None, None)
        assert rc == 1
    arr = (ctypes.c_int * 3)(0, 5, 9)
    assert lib.gdn_prefill_varlen(ctypes.byref(s), 2, None, arr, None, None, None, None, 0x900000, 0x2000000,
                                  1 << 30, None, None) == 1


def test_decode_rejects_aliasing(lib):
    s = fake_inputs()
    assert lib.gdn_decode_step(ctypes.byref(s), 4, 0x7000000, 0x7000000 + 64, 0x900000, None, None) == 4
    assert lib.gdn_decode_step(ctypes.byref(s), 4, None, 0x7000000, 0x900000, None, None) == 1
    assert lib.gdn_decode_step(ctypes.byref(s), 0, None, None, None, None, None) == 0


def test_decode_multi_rejects_bad_arguments(lib):
    s = fake_inputs()
    st, cv, out = 0x7000000, 0x5000000, 0x900000
    # T outside 1 .. GDN_MAX_DECODE_TOKENS, negative N or pool size
    for T in (0, gdn.MAX_DECODE_TOKENS + 1):
        assert lib.gdn_decode_multi(ctypes.byref(s), 2, T, st, cv, None, 2, out, None, None) == 1
    assert lib.gdn_decode_multi(ctypes.byref(s), -1, 1, st, cv, None, 2, out, None, None) == 1
    assert lib.gdn_decode_multi(ctypes.byref(s), 2, 1, st, cv, 0x3000000, -1, out, None, None) == 1
    # without slots sequence n uses slot n, so the pool must hold N states
    assert lib.gdn_decode_multi(ctypes.byref(s), 3, 1, st, cv, None, 2, out, None, None) == 1
    # a misaligned slot array, a state overlapping the output
    assert lib.gdn_decode_multi(ctypes.byref(s), 2, 2, st, cv, 0x3000002, 4, out, None, None) == 3
    assert lib.gdn_decode_multi(ctypes.byref(s), 2, 2, st, cv, None, 2, st + 1024, None, None) == 4
    # N = 0 is a no-op
    assert lib.gdn_decode_multi(ctypes.byref(s), 0, 4, None, None, None, 0, None, None, None) == 0


def test_layer_sizes_and_rejections(lib):
    assert lib.gdn_layer_n_in(16, 48) == 2 * 16 * 128 + 2 * 48 * 128 + 2 * 48 == 16480
    assert lib.gdn_layer_n_in(2, 6) == 2060 and lib.gdn_layer_n_in(0, 6) == 0
    T = 4096
    want = (-(-T * 16480 * 2 // 1024) * 1024) + (-(-T * 6144 * 2 // 1024) * 1024) + \
        lib.gdn_prefill_workspace_size(16, 48, 1, T // 64)
    assert lib.gdn_layer_workspace_size(16, 48, 1, T) == want
    L = gdn.GdnLayer()
    L.w_in, L.ld_w_in, L.w_out, L.ld_w_out = 0x100000, 5120, 0x200000, 6144
    L.conv_w, L.A_log, L.norm_w = 0x300000, 0x310000, 0x320000
    L.H_k, L.H_v, L.hidden, L.scale = 16, 48, 5120, 1.0
    args = (1, 64, 0x400000, 5120, None, None, None, None, 0x900000, 5120, 0x2000000, 1 << 31, None, None)
    L.hidden = 5000  # not a multiple of 64
    assert lib.gdn_layer_prefill(ctypes.byref(L), *args) == 2
    L.hidden = 5120
    assert lib.gdn_layer_prefill(ctypes.byref(L), 1, 64, None, *args[3:]) == 1
    small = args[:11] + (1024,) + args[12:]
    assert lib.gdn_layer_prefill(ctypes.byref(L), *small) == 7
    assert lib.gdn_layer_prefill(ctypes.byref(L), 0, 64, *args[2:]) == 0
    # state and conv checks come before the input projection is launched
    # (args: B, T, x, ldx, state_in, state_out, conv_in, conv_out, y, ldy, workspace, bytes, err, stream)
    def with_(**kw):
        a = list(args)
        for k, val in kw.items():
            a[int(k[1:])] = val
        return lib.gdn_layer_prefill(ctypes.byref(L), *a)
    assert with_(i4=0x40000000, i5=0x40000000 + 4096) == 4       # state_in, state_out overlapping, not equal
    assert with_(i6=0x50000000, i7=0x50000000) == 4              # conv_out == conv_in
    assert with_(i4=0x40000000, i6=0x40000000) == 4              # state and conv history in the same place
    assert with_(i4=0x40000008) == 3                             # misaligned state_in
    assert with_(i5=0x2000000 + 8192) == 4                       # state_out inside the workspace
    # what the mixer call would reject is rejected before the input projection is launched
    # (on this GPU-less host a launch would fail with GDN_ERR_CUDA = 5 instead)
    L.H_k, L.H_v = 1, 16                                         # 16 value heads per key head
    assert lib.gdn_layer_prefill(ctypes.byref(L), *args) == 2
    L.H_k, L.H_v = 16, 48
    L.conv_w = None
    assert lib.gdn_layer_prefill(ctypes.byref(L), *args) == 1
    L.conv_w = 0x300008                                          # misaligned conv weights
    assert lib.gdn_layer_prefill(ctypes.byref(L), *args) == 3
    L.conv_w = 0x300000


def _attn_layer(hidden=5120):
    L = gdn.GdnAttnLayer()
    L.w_in, L.ld_w_in, L.w_out, L.ld_w_out = 0x100000, hidden, 0x8000000, 24 * 256
    L.q_norm_w, L.k_norm_w, L.hidden = 0x10000000, 0x10001000, hidden
    return L


def test_attention_sizes_and_rejections(lib):
    up = lambda n: -(-n // 1024) * 1024
    n_in, hd = 2 * 24 * 256 + 2 * 4 * 256, 24 * 256
    assert lib.gdn_attn_layer_workspace_size(2, 100) == up(200 * n_in * 2) + 2 * up(200 * hd * 2)
    assert lib.gdn_attn_layer_workspace_size(-1, 100) == 0
    # decode: projection, q_hat, attention output, then fp32 partials (o[256], m, l) per
    # (sequence, KV head, split of 512 cache rows, query head of the group)
    for N, cap in ((64, 4096), (3, 153), (1, 513)):
        parts = N * 4 * (-(-cap // 512)) * 6 * 258 * 4
        assert lib.gdn_attn_decode_workspace_size(N, cap) == up(N * n_in * 2) + 2 * up(N * hd * 2) + up(parts)
    assert lib.gdn_attn_decode_workspace_size(4, -1) == 0

    L = _attn_layer()
    B, T, cap = 1, 256, 512
    ws_bytes = lib.gdn_attn_layer_workspace_size(B, T)
    # x, k_cache, v_cache, cache_cap, y, ldy, workspace, bytes, err, stream
    ok_args = [0x20000000, 5120, 0x30000000, 0x40000000, cap, 0x50000000, 5120, 0x60000000, ws_bytes, None, None]
    bad = lambda **kw: [kw.get(str(i), a) for i, a in enumerate(ok_args)]
    prefill = lambda L, B, T, args: lib.gdn_attn_layer_prefill(ctypes.byref(L), B, T, *args)
    assert prefill(L, -1, T, ok_args) == 1                       # bad count
    assert prefill(L, B, T, bad(**{"4": 100})) == 1              # cache smaller than the prompt
    assert prefill(L, B, T, bad(**{"0": None})) == 1             # null input
    assert prefill(L, B, T, bad(**{"8": ws_bytes - 1})) == 7     # workspace too small
    assert prefill(L, B, T, bad(**{"2": 0x30000008})) == 3       # misaligned K cache
    assert prefill(L, B, T, bad(**{"7": 0x50000000})) == 4       # workspace overlaps y
    assert prefill(L, 0, T, ok_args) == 0                        # nothing to do, nothing launched
    assert prefill(_attn_layer(5000), B, T, ok_args) == 2        # hidden not a multiple of 64

    N = 4
    dws = lib.gdn_attn_decode_workspace_size(N, cap)
    # x, ldx, k_cache, v_cache, cache_cap, cache_len, y, ldy, workspace, bytes, err, stream
    d_args = [0x20000000, 5120, 0x30000000, 0x40000000, cap, 0x70000000, 0x50000000, 5120, 0x60000000, dws, None,
              None]
    dbad = lambda **kw: [kw.get(str(i), a) for i, a in enumerate(d_args)]
    step = lambda N, args: lib.gdn_attn_layer_decode_step(ctypes.byref(L), N, *args)
    assert step(N, dbad(**{"4": 0})) == 1                        # no cache
    assert step(N, dbad(**{"5": None})) == 1                     # no cache_len
    assert step(N, dbad(**{"9": dws - 1})) == 7                  # workspace too small
    assert step(N, dbad(**{"3": 0x40000004})) == 3               # misaligned V cache
    assert step(0, d_args) == 0                                  # no sequences, nothing launched


def test_prefill_host_sizes_and_rejections(lib):
    up = lambda n: -(-n // 1024) * 1024
    H_k, H_v, B, T = 16, 48, 2, 100
    T_tot, C_conv = B * T, (2 * H_k + H_v) * 128
    base = up(lib.gdn_prefill_workspace_size(H_k, H_v, B, B * 2))
    staged = 2 * up(T_tot * H_k * 128 * 2) + 3 * up(T_tot * H_v * 128 * 2) + 2 * up(T_tot * H_v * 2) + \
        up(B * H_v * 128 * 128 * 4) + 2 * up(B * 3 * C_conv * 2)
    need = lib.gdn_prefill_host_workspace_size(H_k, H_v, B, T)
    assert need == base + staged
    assert lib.gdn_prefill_host_workspace_size(H_k, H_v, -1, T) == 0
    s = gdn.GdnInputs()
    s.q, s.k, s.v, s.a, s.b, s.z = 0x1000000, 0x2000000, 0x3000000, 0x4000000, 0x5000000, 0x6000000
    s.stride_q, s.stride_k, s.stride_v, s.stride_z, s.stride_a, s.stride_b = 2048, 2048, 6144, 6144, 48, 48
    s.conv_w, s.A_log, s.norm_w = 0x7000000, 0x7100000, 0x7200000
    s.H_k, s.H_v, s.scale = H_k, H_v, 1.0
    # state_in, state_out, conv_in, conv_out, out, workspace, bytes, err, stream
    args = [None, None, None, None, 0x8000000, 0x10000000, need, None, None]
    call = lambda B, a: lib.gdn_prefill_host(ctypes.byref(s), B, T, *a)
    assert call(-1, args) == 1
    assert call(B, args[:4] + [None] + args[5:]) == 1            # no output
    assert call(B, args[:6] + [need - 1] + args[7:]) == 7        # workspace too small
    assert call(B, args[:4] + [0x3000000] + args[5:]) == 4       # output over the v input
    assert call(B, args[:5] + [0x10000008] + args[6:]) == 3      # misaligned workspace
    assert call(0, args) == 0                                    # nothing to do


def test_layer_decode_sizes_and_rejections(lib):
    up = lambda n: -(-n // 1024) * 1024
    assert lib.gdn_layer_decode_workspace_size(16, 48, 256, 1) == up(256 * 16480 * 2) + up(256 * 6144 * 2)
    assert lib.gdn_layer_decode_workspace_size(16, 48, 4, 9) == 0 and lib.gdn_layer_decode_workspace_size(16, 48, 4, 0) == 0
    L = gdn.GdnLayer()
    L.w_in, L.ld_w_in, L.w_out, L.ld_w_out = 0x100000, 5120, 0x20000000, 6144
    L.conv_w, L.A_log, L.norm_w = 0x300000, 0x310000, 0x320000
    L.H_k, L.H_v, L.hidden, L.scale = 16, 48, 5120, 1.0
    N, T = 4, 2
    need = lib.gdn_layer_decode_workspace_size(16, 48, N, T)
    # x, ldx, state, conv_state, state_slot, n_slots, y, ldy, workspace, bytes, err, stream
    args = [0x400000, 5120, 0x40000000, 0x50000000, None, 0, 0x900000, 5120, 0x60000000, need, None, None]
    call = lambda N, T, a: lib.gdn_layer_decode(ctypes.byref(L), N, T, *a)
    assert call(N, 0, args) == 1 and call(N, 9, args) == 1      # tokens per call out of range
    assert call(N, T, args[:9] + [need - 1] + args[10:]) == 7    # workspace too small
    assert call(N, T, args[:6] + [0x60000000] + args[7:]) == 4   # y inside the workspace
    assert call(N, T, [None] + args[1:]) == 1                    # no input
    assert call(N, T, args[:2] + [None] + args[3:]) == 1         # no state: rejected before any launch
    assert call(N, T, args[:2] + [0x40000004] + args[3:]) == 3   # misaligned state
    assert call(N, T, args[:3] + [0x40000000 + 1024] + args[4:]) == 4  # conv state inside the state pool
    assert call(0, T, args) == 0                                 # no sequences, nothing launched
    assert call(N, T, args[:2] + [0x60000000 + 2048] + args[3:]) == 4  # state inside the workspace
    L.H_k, L.H_v = 1, 16                                         # decode-call rejections come first too
    assert call(N, T, args) == 2
    L.H_k, L.H_v = 16, 48
    L.norm_w = None
    assert call(N, T, args) == 1
    L.norm_w = 0x320000
    L.hidden = 5000
    assert call(N, T, args) == 2


def test_fused_plan_follows_the_available_sms(lib):
    """The overlapped prefill launch is chosen from the SMs the context may use: its scan CTAs
    (N * H_v) must fit in half of them, and the automatic plan also wants >= 8 prep items per
    remaining SM; a partition of the device (a green context, an MPS share) with fewer SMs
    falls back to two launches instead of leaving the scan waiting for a prep with no SM."""
    plan = lib.gdn_prefill_fused_plan
    # one 4096-token prompt, 16 / 48 heads: 64 chunks x 16 key heads = 1024 prep items
    assert plan(16, 48, 1, 64, 0, 148) == 48
    assert plan(16, 48, 1, 64, 2, 148) == 48
    assert plan(16, 48, 1, 64, 1, 148) == 0          # two launches asked for
    assert plan(16, 48, 1, 64, 0, 95) == 0           # 48 scan CTAs need 96 SMs
    assert plan(16, 48, 1, 64, 2, 96) == 48
    assert plan(16, 48, 1, 8, 0, 148) == 0           # 128 items: too few for the other 100 SMs
    assert plan(16, 48, 1, 8, 2, 148) == 48          # forced: fused all the same
    assert plan(16, 48, 8, 1681, 0, 148) == 0        # 8 sequences: 384 scan units, two launches
    assert plan(2, 6, 1, 8, 2, 148) == 6
    assert plan(16, 48, 1, 64, 0, 0) == 0 and plan(0, 48, 1, 64, 0, 148) == 0


def test_nvtx_ranges_switch_on_from_the_environment():
    """GDN_NVTX=1: the entry points push NVTX ranges (no profiler attached, so no-ops); a call
    that fails validation still returns its status and pops its range."""
    import subprocess
    import sys
    code = (
        "import ctypes, sys; sys.path.insert(0, %r)\n"
        "from gated_delta_rule_81_b200 import gdn\n"
        "lib = gdn.load()\n"
        "s = gdn.GdnInputs()\n"
        "rc = lib.gdn_prefill(ctypes.byref(s), -1, 4, None, None, None, None, None, None, 0, None, None)\n"
        "rc2 = lib.gdn_decode_step(ctypes.byref(s), -1, None, None, None, None, None)\n"
        "print(rc, rc2)\n" % ROOT)
    env = dict(os.environ, GDN_NVTX="1")
    r = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr
    assert r.stdout.split() == ["1", "1"]  # GDN_ERR_INVALID_ARG, from both
