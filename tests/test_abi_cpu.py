"""The C-ABI library on a machine without a GPU: it loads, exports every
function include/lb.h declares, answers the host-only queries, and rejects bad
arguments before it touches CUDA.  No call here reaches a kernel."""
import ctypes
import re

import pytest

import binarized_rank_linear_b200 as lb
import oracle
from binarized_rank_linear_b200 import build as lb_build
from binarized_rank_linear_b200 import synth


@pytest.fixture(scope="module")
def L():
    lb_build.build()
    return lb.lib()


def declared_functions():
    text = open(lb.HEADER_PATH).read()
    return sorted(set(re.findall(r"LB_API\s+[\w\s\*]+?\b(lb_\w+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("lb_pack_signs", "lb_linear_forward", "lb_rank_for_budget", "lb_packed_ld_words",
                     "lb_packed_bytes", "lb_forward_workspace_bytes", "lb_device_status",
                     "lb_status_string"):
        assert required in names


def test_every_declared_symbol_is_exported(L):
    for name in declared_functions():
        assert hasattr(L, name), f"{name} missing from {lb.LIB_PATH}"


def test_status_strings(L):
    for code in range(0, 9):
        s = lb.status_string(code)
        assert s.startswith("LB_") and "UNKNOWN" not in s
    assert lb.status_string(99) == "LB_ERR_UNKNOWN"


def test_packed_ld_and_bytes_match_the_oracle_packer(L):
    for cols in (1, 31, 32, 33, 288, 800, 1024, 4096, 11008, 28672):
        assert lb.packed_ld_words(cols) == -(-cols // 32)
    assert lb.packed_ld_words(0) == -1
    assert lb.packed_bytes(lb.LB_FACTOR_U, 28672, 288) == 28672 * 9 * 4
    assert lb.packed_bytes(lb.LB_FACTOR_V, 8192, 288) == 288 * 256 * 4
    assert lb.packed_bytes(lb.LB_FACTOR_U, 0, 32) == 0


@pytest.mark.parametrize("name", sorted(synth.CONFIGS))
def test_rank_rule_matches_oracle_and_table(L, name):
    c = synth.CONFIGS[name]
    r = lb.rank_for_budget(c.n_in, c.n_out, c.eff_num, c.eff_den, c.paths, 32)
    assert r == c.rank == oracle.rank_for_budget(c.n_in, c.n_out, c.eff_num, c.eff_den, c.paths, 32)


def test_rank_rule_random_against_oracle(L):
    import random
    rnd = random.Random(3)
    for _ in range(500):
        n_in, n_out = rnd.randint(1, 1 << 18), rnd.randint(1, 1 << 18)
        num, den = rnd.randint(1, 200), rnd.randint(1, 200)
        paths, align = rnd.choice([1, 2]), rnd.choice([1, 8, 32, 64])
        expect = oracle.rank_for_budget(n_in, n_out, num, den, paths, align)
        r = ctypes.c_int64(-1)
        st = L.lb_rank_for_budget(n_in, n_out, num, den, paths, align, ctypes.byref(r))
        assert r.value == expect
        assert st == (lb.LB_OK if expect > 0 else lb.LB_ERR_UNSUPPORTED_SHAPE)


def test_rank_rule_rejects_bad_arguments(L):
    r = ctypes.c_int64(5)
    assert L.lb_rank_for_budget(0, 10, 1, 1, 1, 1, ctypes.byref(r)) == lb.LB_ERR_INVALID_ARGUMENT
    assert L.lb_rank_for_budget(10, 10, 1, 1, 3, 1, ctypes.byref(r)) == lb.LB_ERR_INVALID_ARGUMENT
    assert L.lb_rank_for_budget(10, 10, 1, 0, 1, 1, ctypes.byref(r)) == lb.LB_ERR_INVALID_ARGUMENT
    assert L.lb_rank_for_budget(10, 10, 1, 1, 1, 1, None) == lb.LB_ERR_INVALID_ARGUMENT
    # no int64 overflow for huge (valid) inputs
    big = 1 << 40
    assert L.lb_rank_for_budget(big, big, 1, 1, 1, 1, ctypes.byref(r)) == lb.LB_OK
    assert r.value == big // 2


def test_workspace_query(L):
    for name in ("tiny", "llama2_7b_q", "llama2_70b_gate"):
        c = synth.CONFIGS[name]
        for m in (1, 8, 32):
            assert lb.forward_workspace_bytes(m, c.n_in, c.n_out, c.rank,
                                              c.rank if c.paths == 2 else 0) > 0
    assert lb.forward_workspace_bytes(0, 256, 256, 32, 0) == 0
    assert lb.forward_workspace_bytes(1, 256, 256, 0, 0) == 0


FAKE = 0x10000          # 16-byte aligned, never dereferenced: every call below fails its checks first


def fake_path(rank=32, **over):
    d = dict(u_bits=FAKE, vt_bits=FAKE, h=FAKE, g=FAKE, l=FAKE, rank=rank, u_ld=0, vt_ld=0)
    d.update(over)
    return lb.LbPath(**d)


def forward(L, x=FAKE, tokens=1, n_in=256, n_out=256, ldx=256, main=None, residual=None, y=FAKE,
            ldy=256, ws=FAKE, ws_bytes=1 << 20):
    main = fake_path() if main is None else main
    return L.lb_linear_forward(x, tokens, n_in, n_out, ldx, ctypes.byref(main),
                               ctypes.byref(residual) if residual is not None else None, y, ldy, ws,
                               ws_bytes, None)


def test_forward_rejects_bad_arguments_before_any_cuda_call(L):
    assert forward(L, tokens=-1) == lb.LB_ERR_INVALID_ARGUMENT
    assert forward(L, tokens=0, x=0, y=0) == lb.LB_OK                 # no-op
    assert forward(L, x=0) == lb.LB_ERR_INVALID_ARGUMENT
    assert forward(L, y=0) == lb.LB_ERR_INVALID_ARGUMENT
    assert forward(L, n_in=250, ldx=256) == lb.LB_ERR_UNSUPPORTED_SHAPE
    assert forward(L, n_out=100, ldy=256) == lb.LB_ERR_UNSUPPORTED_SHAPE
    assert forward(L, ldx=128) == lb.LB_ERR_INVALID_ARGUMENT
    assert forward(L, ldx=260) == lb.LB_ERR_MISALIGNED
    assert forward(L, x=FAKE + 2) == lb.LB_ERR_MISALIGNED
    assert forward(L, main=fake_path(rank=48)) == lb.LB_ERR_UNSUPPORTED_SHAPE
    assert forward(L, main=fake_path(rank=0)) == lb.LB_ERR_INVALID_ARGUMENT
    assert forward(L, main=fake_path(u_bits=0)) == lb.LB_ERR_INVALID_ARGUMENT
    assert forward(L, main=fake_path(g=FAKE + 4)) == lb.LB_ERR_MISALIGNED
    assert forward(L, main=fake_path(vt_ld=7)) == lb.LB_ERR_INVALID_ARGUMENT   # < ceil(256/32)
    assert forward(L, residual=fake_path(l=0)) == lb.LB_ERR_INVALID_ARGUMENT
    assert forward(L, ws_bytes=16) == lb.LB_ERR_WORKSPACE_TOO_SMALL
    assert forward(L, ws=0) == lb.LB_ERR_INVALID_ARGUMENT
    assert forward(L, ws=FAKE + 8) == lb.LB_ERR_MISALIGNED


def test_pack_rejects_bad_arguments_before_any_cuda_call(L):
    P = L.lb_pack_signs
    assert P(0, lb.LB_I8, lb.LB_FACTOR_U, 4, 32, 32, FAKE, 1, None) == lb.LB_ERR_INVALID_ARGUMENT
    assert P(FAKE, 9, lb.LB_FACTOR_U, 4, 32, 32, FAKE, 1, None) == lb.LB_ERR_INVALID_ARGUMENT
    assert P(FAKE, lb.LB_I8, 5, 4, 32, 32, FAKE, 1, None) == lb.LB_ERR_INVALID_ARGUMENT
    assert P(FAKE, lb.LB_I8, lb.LB_FACTOR_U, 4, 32, 16, FAKE, 1, None) == lb.LB_ERR_INVALID_ARGUMENT
    assert P(FAKE, lb.LB_I8, lb.LB_FACTOR_U, 4, 64, 64, FAKE, 1, None) == lb.LB_ERR_INVALID_ARGUMENT
    assert P(FAKE, lb.LB_I8, lb.LB_FACTOR_V, 64, 32, 32, FAKE, 1, None) == lb.LB_ERR_INVALID_ARGUMENT
    assert P(FAKE + 1, lb.LB_F32, lb.LB_FACTOR_U, 4, 32, 32, FAKE, 1, None) == lb.LB_ERR_MISALIGNED
    assert P(FAKE, lb.LB_F32, lb.LB_FACTOR_U, 4, 32, 32, FAKE + 2, 1, None) == lb.LB_ERR_MISALIGNED


def forward_fixed(L, x=FAKE, tokens=1, n_in=256, n_out=256, ldx=256, main=None, residual=None, y=FAKE,
                  ldy=256):
    main = fake_path() if main is None else main
    return L.lb_linear_forward_fixed_scratch(x, tokens, n_in, n_out, ldx, ctypes.byref(main),
                                             ctypes.byref(residual) if residual is not None else None,
                                             y, ldy, None)


def test_fixed_scratch_rejects_before_any_cuda_call(L):
    """The fixed-scratch entry serves 1..32 tokens and shapes whose scratch
    fits LB_FIXED_SCRATCH_BYTES (1 MiB); everything else is refused on the
    host, before the device is touched."""
    assert forward_fixed(L, tokens=0) == lb.LB_OK
    assert forward_fixed(L, tokens=-1) == lb.LB_ERR_INVALID_ARGUMENT
    assert forward_fixed(L, tokens=33) == lb.LB_ERR_UNSUPPORTED_SHAPE
    assert forward_fixed(L, x=0) == lb.LB_ERR_INVALID_ARGUMENT
    assert forward_fixed(L, y=0) == lb.LB_ERR_INVALID_ARGUMENT
    assert L.lb_linear_forward_fixed_scratch(FAKE, 1, 256, 256, 256, None, None, FAKE, 256,
                                             None) == lb.LB_ERR_INVALID_ARGUMENT
    # two rank-32768 paths at 32 tokens need 4 MiB of latent scratch
    big = fake_path(rank=32768)
    assert L.lb_forward_workspace_bytes(32, 4096, 4096, 32768, 32768) > (1 << 20)
    assert forward_fixed(L, tokens=32, n_in=4096, n_out=4096, ldx=4096, ldy=4096, main=big,
                         residual=big) == lb.LB_ERR_WORKSPACE_TOO_SMALL


def test_split_halves_reject_bad_arguments_before_any_cuda_call(L):
    """lb_latent_forward checks the V half of each path and lb_expand_forward
    the U half; the other half may be null.  Everything is refused on the
    host before the device is touched."""
    lat = lambda **kw: L.lb_latent_forward(
        kw.get("x", FAKE), kw.get("tokens", 1), kw.get("n_in", 256), kw.get("ldx", 256),
        ctypes.byref(kw.get("main", fake_path(u_bits=0, h=0))), None, kw.get("z", FAKE), kw.get("ldz", 32), None)
    exp = lambda **kw: L.lb_expand_forward(
        kw.get("z", FAKE), kw.get("tokens", 1), kw.get("n_out", 256), kw.get("ldz", 32),
        ctypes.byref(kw.get("main", fake_path(vt_bits=0, g=0, l=0))), None, kw.get("y", FAKE), kw.get("ldy", 256),
        None)
    for f in (lat, exp):
        assert f(tokens=0) == lb.LB_OK
        assert f(tokens=-1) == lb.LB_ERR_INVALID_ARGUMENT
        assert f(z=0) == lb.LB_ERR_INVALID_ARGUMENT
        assert f(ldz=16) == lb.LB_ERR_INVALID_ARGUMENT          # below the rank
        assert f(ldz=36) == lb.LB_ERR_MISALIGNED                 # not a multiple of 8
        assert f(z=FAKE + 2) == lb.LB_ERR_MISALIGNED
        assert f(main=fake_path(rank=48)) == lb.LB_ERR_UNSUPPORTED_SHAPE
    assert lat(x=0) == lb.LB_ERR_INVALID_ARGUMENT
    assert lat(n_in=48, ldx=48) == lb.LB_ERR_UNSUPPORTED_SHAPE
    assert lat(main=fake_path(g=0)) == lb.LB_ERR_INVALID_ARGUMENT  # the V half is required
    assert lat(main=fake_path(vt_bits=FAKE + 4)) == lb.LB_ERR_MISALIGNED
    assert exp(y=0) == lb.LB_ERR_INVALID_ARGUMENT
    assert exp(n_out=48, ldy=48) == lb.LB_ERR_UNSUPPORTED_SHAPE
    assert exp(main=fake_path(h=0)) == lb.LB_ERR_INVALID_ARGUMENT  # the U half is required
    assert exp(main=fake_path(u_bits=FAKE + 4)) == lb.LB_ERR_MISALIGNED


def siblings(L, projs=None, nproj=None, x=FAKE, tokens=1, n_in=256, ldx=256, ws=FAKE, ws_bytes=1 << 20):
    """lb_linear_forward_siblings over fake projections [(n_out, main, residual, y, ldy), ...]."""
    projs = [(256, fake_path(), None, FAKE, 256), (96, fake_path(64), fake_path(), FAKE, 96)] if projs is None else projs
    arr = (lb.LbProjection * max(1, len(projs)))()
    keep = []
    for j, (n_out, main, res, y, ldy) in enumerate(projs):
        keep += [main, res]
        arr[j].n_out, arr[j].y, arr[j].ldy = n_out, y, ldy
        arr[j].main = ctypes.pointer(main) if main is not None else None
        arr[j].residual = ctypes.pointer(res) if res is not None else None
    return L.lb_linear_forward_siblings(x, tokens, n_in, ldx, len(projs) if nproj is None else nproj,
                                        arr, ws, ws_bytes, None)


def test_siblings_reject_bad_arguments_before_any_cuda_call(L):
    assert siblings(L, tokens=0, x=0) == lb.LB_OK                       # no-op
    assert siblings(L, tokens=-1) == lb.LB_ERR_INVALID_ARGUMENT
    assert siblings(L, nproj=0) == lb.LB_ERR_INVALID_ARGUMENT
    assert siblings(L, nproj=lb.MAX_SIBLINGS + 1) == lb.LB_ERR_INVALID_ARGUMENT
    assert siblings(L, x=0) == lb.LB_ERR_INVALID_ARGUMENT
    assert siblings(L, x=FAKE + 2) == lb.LB_ERR_MISALIGNED
    assert siblings(L, n_in=250, ldx=256) == lb.LB_ERR_UNSUPPORTED_SHAPE
    bad = lambda **kw: [(256, fake_path(), None, FAKE, 256), (kw.get("n_out", 96), kw.get("main", fake_path()),
                                                             kw.get("res", None), kw.get("y", FAKE), kw.get("ldy", 96))]
    assert siblings(L, bad(n_out=100, ldy=104)) == lb.LB_ERR_UNSUPPORTED_SHAPE
    assert siblings(L, bad(main=None)) == lb.LB_ERR_INVALID_ARGUMENT
    assert siblings(L, bad(y=0)) == lb.LB_ERR_INVALID_ARGUMENT
    assert siblings(L, bad(y=FAKE + 2)) == lb.LB_ERR_MISALIGNED
    assert siblings(L, bad(ldy=64)) == lb.LB_ERR_INVALID_ARGUMENT
    assert siblings(L, bad(ldy=100)) == lb.LB_ERR_MISALIGNED
    assert siblings(L, bad(main=fake_path(rank=48))) == lb.LB_ERR_UNSUPPORTED_SHAPE
    assert siblings(L, bad(res=fake_path(h=0))) == lb.LB_ERR_INVALID_ARGUMENT
    assert siblings(L, ws_bytes=16) == lb.LB_ERR_WORKSPACE_TOO_SMALL
    assert siblings(L, ws=0) == lb.LB_ERR_INVALID_ARGUMENT
    assert siblings(L, ws=FAKE + 8) == lb.LB_ERR_MISALIGNED


def test_siblings_workspace_covers_each_layer_and_the_group(L):
    """The group's workspace is at least each projection's own (the paths
    that run one layer at a time) and, for 1..4 tokens, the fp32 latent of
    every path of the group."""
    q, kv = synth.CONFIGS["qwen3_14b_qo"], synth.CONFIGS["qwen3_14b_kv"]
    layers = [(q.n_out, q.rank), (kv.n_out, kv.rank), (kv.n_out, kv.rank)]
    arr = (lb.LbProjection * 3)()
    keep = []
    for j, (n_out, r) in enumerate(layers):
        m, res = fake_path(r), fake_path(r)
        keep += [m, res]
        arr[j].n_out, arr[j].main, arr[j].residual = n_out, ctypes.pointer(m), ctypes.pointer(res)
    for tokens in (1, 4, 5, 40, 300):
        need = L.lb_siblings_workspace_bytes(tokens, q.n_in, 3, arr)
        for n_out, r in layers:
            assert need >= lb.forward_workspace_bytes(tokens, q.n_in, n_out, r, r)
        if tokens <= 4:
            assert need >= 4 * tokens * sum(2 * r for _, r in layers)
    assert L.lb_siblings_workspace_bytes(0, q.n_in, 3, arr) == 0
    assert L.lb_siblings_workspace_bytes(1, q.n_in, 0, arr) == 0
    assert L.lb_siblings_workspace_bytes(1, 250, 3, arr) == 0


def test_host_buffer_call_rejects_before_any_cuda_call(L):
    host = lambda **kw: L.lb_linear_forward_host(
        kw.get("xh", FAKE), kw.get("tokens", 1), kw.get("n_in", 256), kw.get("n_out", 256),
        ctypes.byref(kw.get("main", fake_path())), None, kw.get("yh", FAKE), kw.get("xd", FAKE), kw.get("yd", FAKE),
        kw.get("ws", FAKE), kw.get("ws_bytes", 1 << 20), None)
    assert host(tokens=0, xh=0, yh=0) == lb.LB_OK            # no-op
    assert host(tokens=-1) == lb.LB_ERR_INVALID_ARGUMENT
    assert host(xh=0) == lb.LB_ERR_INVALID_ARGUMENT
    assert host(yh=0) == lb.LB_ERR_INVALID_ARGUMENT
    assert host(xd=0) == lb.LB_ERR_INVALID_ARGUMENT
    assert host(yd=FAKE + 2) == lb.LB_ERR_MISALIGNED
    assert host(n_in=250) == lb.LB_ERR_UNSUPPORTED_SHAPE
    assert host(main=fake_path(rank=48)) == lb.LB_ERR_UNSUPPORTED_SHAPE
    assert host(ws_bytes=16) == lb.LB_ERR_WORKSPACE_TOO_SMALL


def test_prefill_pairs_switch_takes_only_zero_or_one(L):
    # host-only: the setting is a process-wide flag read when a call plans its tiles
    for bad in (-1, 2, 7):
        assert L.lb_set_prefill_pairs(bad) == lb.LB_ERR_INVALID_ARGUMENT
    assert L.lb_set_prefill_pairs(0) == lb.LB_OK
    assert L.lb_set_prefill_pairs(1) == lb.LB_OK


def test_binding_rejects_wrong_dtype_or_layout_before_any_call(L):
    """The binding checks each activation's dtype, rank and inner stride (and
    that it lives on the device) before its pointer reaches the library: an
    fp16 tensor or a transposed view would otherwise be read as wrong bits."""
    import torch
    fake = lb.PackedPath(torch.zeros((64, 1), dtype=torch.int32), torch.zeros((32, 2), dtype=torch.int32),
                         torch.zeros(64, dtype=torch.float16), torch.zeros(64, dtype=torch.float16),
                         torch.zeros(32, dtype=torch.float16), 32)
    with pytest.raises(TypeError, match="bfloat16"):
        lb.linear_forward(torch.zeros((2, 64), dtype=torch.float16), fake)
    with pytest.raises(ValueError, match="inner stride"):
        lb.linear_forward(torch.zeros((64, 2), dtype=torch.bfloat16).t(), fake)
    with pytest.raises(ValueError, match="device memory"):
        lb.linear_forward(torch.zeros((2, 64), dtype=torch.bfloat16), fake)
    with pytest.raises(TypeError, match="float16"):
        lb.expand_forward(torch.zeros((2, 32), dtype=torch.bfloat16), fake)
    with pytest.raises(TypeError, match="bfloat16"):
        lb.latent_forward(torch.zeros((2, 64), dtype=torch.float32), fake)
    with pytest.raises(TypeError, match="bfloat16"):
        lb.linear_forward_siblings(torch.zeros((2, 64), dtype=torch.float16), [(fake, None)])
    with pytest.raises(TypeError, match="bfloat16"):
        lb.linear_forward_fixed_scratch(torch.zeros((2, 64), dtype=torch.int16), fake)
    xh = torch.zeros((2, 64), dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="inner stride"):
        lb.linear_forward_host(torch.zeros((64, 2), dtype=torch.bfloat16).t(), fake, None,
                               torch.zeros((2, 64), dtype=torch.bfloat16), xh, xh, torch.zeros(16, dtype=torch.uint8))
    with pytest.raises(ValueError, match="int32"):
        lb.PackedPath(fake.u_bits.float(), fake.vt_bits, fake.h, fake.g, fake.l, 32).as_c()


def test_backward_workspace_and_host_refusals(L):
    """lb_backward_workspace_bytes answers on the host; lb_linear_backward
    refuses bad arguments before it touches CUDA (no device here)."""
    import ctypes
    R, M, n_in, n_out = 2 * 1088, 8192, 5120, 17408
    need = lb.backward_workspace_bytes(M, n_in, n_out, 1088, 1088)
    # transposed signs, c and a in fp16, and fp32 partials per 32-token block
    assert need >= 2 * 1088 * (n_in + n_out) // 8 + 2 * M * R * 2 + (M // 32) * (R + 2 * n_out + 2 * n_in) * 4
    assert lb.backward_workspace_bytes(0, n_in, n_out, 1088, 1088) == 0
    assert lb.backward_workspace_bytes(M, 100, n_out, 1088, 0) == 0
    fake = ctypes.c_void_p(1 << 20)
    p = lb.LbPath(1 << 20, 1 << 20, 1 << 20, 1 << 20, 1 << 20, 32, 0, 0)
    args = lambda **k: [k.get("x", fake), fake, 8, k.get("n_in", 64), 64, k.get("ldx", 64), 64, ctypes.byref(p), None,
                        fake, 64, k.get("dh", fake), fake, fake, fake, 1 << 30, None]
    assert L.lb_linear_backward(*args(x=None)) == lb.LB_ERR_INVALID_ARGUMENT
    assert L.lb_linear_backward(*args(dh=None)) == lb.LB_ERR_INVALID_ARGUMENT
    assert L.lb_linear_backward(*args(n_in=48, ldx=48)) == lb.LB_ERR_UNSUPPORTED_SHAPE
    assert L.lb_linear_backward(*args(ldx=60)) == lb.LB_ERR_INVALID_ARGUMENT
    assert L.lb_linear_backward(*args(x=ctypes.c_void_p((1 << 20) + 2))) == lb.LB_ERR_MISALIGNED


def test_fault_hook_arguments(L):
    assert L.lb_debug_inject_stall(2, 1000000) == lb.LB_ERR_INVALID_ARGUMENT
    assert L.lb_debug_inject_stall(1, 999) == lb.LB_ERR_INVALID_ARGUMENT
    assert L.lb_debug_inject_stall(1, 3_000_000_000) == lb.LB_ERR_INVALID_ARGUMENT
    assert L.lb_debug_inject_stall(1, 1_000_000) == lb.LB_OK
    assert L.lb_debug_inject_stall(0, 0) == lb.LB_OK
