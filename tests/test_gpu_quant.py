"""GPU parity of the HBM-bound kernels against the oracle, bit for bit:
amax + 16-slot ring descales, per-tensor e4m3 quantization, and the
per-token-group quantizer, on the workloads' shapes and edge cases."""
import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu

fv = pytest.importorskip("fp8_quantized_vit_b200")


def _dev_bf16(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def _host_u8(t: torch.Tensor) -> np.ndarray:
    return t.view(torch.uint8).cpu().numpy()


def _f32_bits(x) -> np.ndarray:
    return np.asarray(x, dtype=np.float32).view(np.uint32)


@pytest.fixture(scope="module")
def ctx():
    assert torch.cuda.is_available()
    return fv.Context()


def _check_ok(ctx):
    st, site = ctx.check()
    assert st == fv.OK, (fv.status_string(st), site)


def test_ring_descales_bit_exact_over_20_forwards(ctx):
    """Dynamic scaling over the 20 forwards of the 8192-token, head_dim-128
    workload: the ring wraps after 16; every forward's descales and the ring
    contents must equal the oracle's bit for bit."""
    w = synth.WORKLOADS["1x8192_d128"]
    ring_d = fv.new_ring()
    desc_d = torch.zeros(3, dtype=torch.float32, device="cuda")
    ring_o = oracle.Ring()
    for f in range(20):
        q, k, v = w.qkv(f)
        amax = [oracle.amax_bf16(x) for x in (q, k, v)]
        want = ring_o.update(amax)
        fv.fp8_amax_ring_update(_dev_bf16(q), _dev_bf16(k), _dev_bf16(v), ring_d, desc_d, ctx=ctx)
        got = desc_d.cpu().numpy()
        assert (_f32_bits(got) == _f32_bits(want)).all(), (f, got, want)
        r = ring_d.cpu().numpy()
        assert (_f32_bits(r[:48].reshape(3, 16)) == _f32_bits(ring_o.hist)).all(), f
        assert r[48:49].view(np.int32)[0] == ring_o.pos[0]
    _check_ok(ctx)


@pytest.mark.parametrize("n", [0, 1, 7, 8, 9, 8 * 1000 + 5, 1 << 20])
def test_amax_ring_ragged_sizes(ctx, n):
    rng = np.random.default_rng(n)
    bits = [np.ascontiguousarray(synth.bf16_tensor(synth.stream_key(n, 0, t), 1, max(n, 1))[0, :n])
            for t in range(3)]
    # put the largest magnitude at the very end so the tail path matters
    if n:
        for t in range(3):
            bits[t][-1] = np.uint16(0xC2F0 + t)  # about -120 with a sign bit
    ring_d = fv.new_ring()
    desc_d = torch.zeros(3, dtype=torch.float32, device="cuda")
    dev = [_dev_bf16(b) if n else torch.empty(8, dtype=torch.bfloat16, device="cuda") for b in bits]
    fv.lib().fp8_amax_ring_update(ctx.handle, dev[0].data_ptr(), dev[1].data_ptr(),
                                  dev[2].data_ptr(), n, ring_d.data_ptr(), desc_d.data_ptr(),
                                  fv._stream())
    ring_o = oracle.Ring()
    want = ring_o.update([oracle.amax_bf16(b) for b in bits])
    assert (_f32_bits(desc_d.cpu().numpy()) == _f32_bits(want)).all()
    _check_ok(ctx)


def test_ring_read_amax(ctx):
    ring_d = fv.new_ring()
    desc_d = torch.zeros(3, dtype=torch.float32, device="cuda")
    seq = [(1.0, 2.0, 3.0), (5.0, 0.5, 0.25), (2.0, 2.0, 2.0)]
    for a in seq:
        x = [torch.full((64,), v, dtype=torch.bfloat16, device="cuda") for v in a]
        fv.fp8_amax_ring_update(*x, ring_d, desc_d, ctx=ctx)
    assert fv.fp8_ring_read_amax(ring_d) == [5.0, 2.0, 3.0]


def _quant_case(ctx, q, k, v, desc):
    n = q.size
    dq, dk, dv = (_dev_bf16(x) for x in (q, k, v))
    d = torch.tensor(desc, dtype=torch.float32, device="cuda")
    outs = [torch.empty(max(n, 8), dtype=torch.uint8, device="cuda") for _ in range(3)]
    fv.lib().fp8_quantize_qkv_per_tensor(ctx.handle, dq.data_ptr(), dk.data_ptr(), dv.data_ptr(),
                                         n, d.data_ptr(), outs[0].data_ptr(),
                                         outs[1].data_ptr(), outs[2].data_ptr(), fv._stream())
    _check_ok(ctx)
    for x, o, s in zip((q, k, v), outs, desc):
        want = oracle.quantize_per_tensor(x.ravel(), s)
        got = _host_u8(o)[:n]
        assert (got == want).all(), (np.nonzero(got != want)[0][:5])


@pytest.mark.parametrize("name", ["1x1024_d72", "1x8192_d128", "3x14400_d72", "3x32400_d72"])
def test_quantize_per_tensor_bit_exact(ctx, name):
    """Static (margin 1.5) and dynamic descales on every workload's tensors."""
    w = synth.WORKLOADS[name]
    q, k, v = w.qkv(0)
    amax = [oracle.amax_bf16(x) for x in (q, k, v)]
    static = [oracle.descale_from_amax(np.float32(1.5) * np.float32(a)) for a in amax]
    _quant_case(ctx, q, k, v, static)
    if name in ("1x1024_d72", "1x8192_d128"):
        tight = [oracle.descale_from_amax(a) for a in amax]  # amax maps onto exactly 448
        _quant_case(ctx, q, k, v, tight)


@pytest.mark.parametrize("n", [1, 7, 8, 9, 4097])
def test_quantize_ragged_and_special_values(ctx, n):
    rng = np.random.default_rng(n)
    base = synth.bf16_tensor(synth.stream_key(5, n, 0), 1, max(n, 1))[0, :n].copy()
    specials = np.array([0x0000, 0x8000, 0x0001, 0x8001, 0x7F7F, 0xFF7F, 0x3F80, 0xBF80],
                        dtype=np.uint16)  # +-0, +-tiny, +-max finite, +-1
    base[: min(n, 8)] = specials[: min(n, 8)]
    for desc in (1.0, 1e-10, 0.013671875, 3.0e-3):
        _quant_case(ctx, base, base[::-1].copy(), base, [desc, desc, desc])


@pytest.mark.parametrize("m,n", [(1, 2048), (37504, 2048), (726, 7168), (4192, 7168),
                                 (8192, 2048), (97200, 1152), (3, 128)])
def test_group_quant_bit_exact(ctx, m, n):
    """Shapes of the group quantizer page's table, and the attention outputs
    of the 8192-token and 3x32400-token workloads."""
    x = synth.bf16_tensor(synth.stream_key(m, n, 7), m, n)
    want_q, want_s = oracle.group_quant(x, 128)
    xd = _dev_bf16(x)
    xq = torch.empty((m, n), dtype=torch.uint8, device="cuda")
    sc = torch.empty((m, n // 128), dtype=torch.float32, device="cuda")
    fv.per_token_group_quant_fp8(xd, 128, xq, sc, ctx=ctx)
    _check_ok(ctx)
    assert (_host_u8(xq) == want_q).all()
    assert (_f32_bits(sc.cpu().numpy()) == _f32_bits(want_s)).all()


@pytest.mark.parametrize("group", [16, 32, 64, 256])
def test_group_quant_other_group_sizes(ctx, group):
    m, n = 129, 1024
    x = synth.bf16_tensor(synth.stream_key(group, 1, 2), m, n)
    x[0, :group] = 0  # an all-zero group takes the 1e-10 floor
    want_q, want_s = oracle.group_quant(x, group)
    xq = torch.empty((m, n), dtype=torch.uint8, device="cuda")
    sc = torch.empty((m, n // group), dtype=torch.float32, device="cuda")
    fv.per_token_group_quant_fp8(_dev_bf16(x), group, xq, sc, ctx=ctx)
    _check_ok(ctx)
    assert (_host_u8(xq) == want_q).all()
    assert (_f32_bits(sc.cpu().numpy()) == _f32_bits(want_s)).all()


def test_amax3_then_ring_push_equals_fused_update(ctx):
    """The split path used when one batch is spread over several GPUs
    (amax, all-reduce, ring push) gives the fused update's bits on one GPU."""
    w = synth.WORKLOADS["1x8192_d128"]
    ring_a, ring_b = fv.new_ring(), fv.new_ring()
    da = torch.zeros(3, dtype=torch.float32, device="cuda")
    db = torch.zeros(3, dtype=torch.float32, device="cuda")
    amax3 = torch.zeros(3, dtype=torch.float32, device="cuda")
    for f in range(18):
        x = [synth.bf16_tensor(synth.stream_key(700 + f, f, t), 512, 2048) for t in range(3)]
        dev = [_dev_bf16(a) for a in x]
        fv.fp8_amax_ring_update(*dev, ring_a, da, ctx=ctx)
        fv.fp8_amax3(*dev, amax3, ctx=ctx)
        assert (_f32_bits(amax3.cpu().numpy()) ==
                _f32_bits([oracle.amax_bf16(a) for a in x])).all()
        fv.fp8_ring_push(amax3, ring_b, db)
        assert (_f32_bits(da.cpu().numpy()) == _f32_bits(db.cpu().numpy())).all(), f
        assert (_f32_bits(ring_a.cpu().numpy()) == _f32_bits(ring_b.cpu().numpy())).all(), f
    _check_ok(ctx)


def _descale_set(n_random: int = 80):
    """Descales that stress the division: the 1e-10 floor, powers of two,
    fp32 values with all-ones mantissas, 448-related values, random ones."""
    f = [1e-10, 2.0 ** -30, 2.0 ** -9, 2.0 ** -1, 1.0, 2.0, 2.0 ** 20,
         np.nextafter(np.float32(1.0), np.float32(0)), np.nextafter(np.float32(2.0), np.float32(0)),
         np.float32(1.0) / np.float32(448.0), np.float32(1.5) / np.float32(448.0),
         np.float32(3.0) / np.float32(7.0), np.float32(0.1), np.float32(1e-3), 0.013671875,
         np.float32(123.456)]
    rng = np.random.default_rng(2025)
    amax = np.exp(rng.uniform(np.log(1e-4), np.log(1e4), n_random)).astype(np.float32)
    f += list(amax / np.float32(448.0))
    return [float(np.float32(v)) for v in f]


def test_quantize_every_bf16_value(ctx):
    """Every finite BF16 value through the per-tensor quantizer at 96
    descales, bit for bit against the oracle's IEEE fp32 division."""
    allb = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    x = allb[(allb & 0x7F80) != 0x7F80]          # drop inf and NaN patterns
    x = np.concatenate([x, x[: (-x.size) % 8]])   # multiple of 8
    for d in _descale_set():
        _quant_case(ctx, x, x[::-1].copy(), x, [d, d, d])


def test_group_quant_every_amax(ctx):
    """Each of the 32640 non-negative finite BF16 values (zero included) is
    the amax of one 128-element group, so the scale amax / 448 and its
    reciprocal are exercised at every value they can take; the other 127
    elements of the group are random BF16 values of magnitude <= the amax,
    either sign.  Bit for bit against the oracle's IEEE division."""
    group = 128
    amax_bits = np.arange(0, 0x7F80, dtype=np.uint32)
    g = amax_bits.size
    rng = np.random.default_rng(2024)
    mag = (rng.random((g, group)) * (amax_bits[:, None] + 1)).astype(np.uint32)
    mag = np.minimum(mag, amax_bits[:, None])
    mag[:, 0] = amax_bits
    sign = rng.integers(0, 2, size=(g, group), dtype=np.uint32) << 15
    x = (mag | sign).astype(np.uint16)
    # the amax element at a random position of its group
    perm = rng.permuted(np.tile(np.arange(group), (g, 1)), axis=1)
    x = np.take_along_axis(x, perm, axis=1)
    x = x.reshape(-1, 8 * group)  # 8 groups per row
    want_q, want_s = oracle.group_quant(x, group)
    xq = torch.empty(x.shape, dtype=torch.uint8, device="cuda")
    sc = torch.empty((x.shape[0], 8), dtype=torch.float32, device="cuda")
    fv.per_token_group_quant_fp8(_dev_bf16(x), group, xq, sc, ctx=ctx)
    _check_ok(ctx)
    got = _host_u8(xq)
    bad = np.nonzero(got != want_q)
    assert bad[0].size == 0, (bad[0][:5], bad[1][:5], got[bad][:5], want_q[bad][:5])
    assert (_f32_bits(sc.cpu().numpy()) == _f32_bits(want_s)).all()


@pytest.mark.parametrize("group", [16, 32, 64, 128, 256])
def test_group_quant_every_bf16_value(ctx, group):
    """Every finite BF16 value (both zeros, subnormals, the largest finite)
    through the group quantizer, shuffled into rows so that groups mix
    magnitudes, bit for bit against the oracle's IEEE division."""
    allb = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    x = allb[(allb & 0x7F80) != 0x7F80]
    rng = np.random.default_rng(group)
    x = rng.permutation(x)
    n = 1024
    x = np.concatenate([x, np.full((-x.size) % n, 0x8000, dtype=np.uint16)]).reshape(-1, n)
    # a few groups of zeros only, of -0 only, and one value among zeros
    x[0, :group] = 0
    x[1, :group] = 0x8000
    x[2, :group] = 0x8000
    x[2, group // 2] = 0x0001
    want_q, want_s = oracle.group_quant(x, group)
    xq = torch.empty(x.shape, dtype=torch.uint8, device="cuda")
    sc = torch.empty((x.shape[0], n // group), dtype=torch.float32, device="cuda")
    fv.per_token_group_quant_fp8(_dev_bf16(x), group, xq, sc, ctx=ctx)
    _check_ok(ctx)
    got = _host_u8(xq)
    bad = np.nonzero(got != want_q)
    assert bad[0].size == 0, (bad[0][:5], bad[1][:5], got[bad][:5], want_q[bad][:5])
    assert (_f32_bits(sc.cpu().numpy()) == _f32_bits(want_s)).all()


def test_fused_amax_ring_quantize_over_20_forwards(ctx):
    """fp8_amax_ring_quantize_qkv (one cooperative launch) over the 20
    forwards of the 8192-token, head_dim-128 workload (the ring wraps after
    16): every forward's descales, ring contents and e4m3 codes equal the
    oracle's ring + quantizer bit for bit, and the two-call path's."""
    w = synth.WORKLOADS["1x8192_d128"]
    n = w.tokens * w.hd
    ring_f, ring_2 = fv.new_ring(), fv.new_ring()
    desc_f = torch.zeros(3, dtype=torch.float32, device="cuda")
    desc_2 = torch.zeros(3, dtype=torch.float32, device="cuda")
    out_f = [torch.empty(n, dtype=torch.uint8, device="cuda") for _ in range(3)]
    out_2 = [torch.empty(n, dtype=torch.uint8, device="cuda") for _ in range(3)]
    ring_o = oracle.Ring()
    for f in range(20):
        x = w.qkv(f)
        dev = [_dev_bf16(a).reshape(-1) for a in x]
        want = ring_o.update([oracle.amax_bf16(a) for a in x])
        fv.fp8_amax_ring_quantize_qkv(*dev, ring_f, desc_f, *out_f, ctx=ctx)
        fv.fp8_amax_ring_update(*dev, ring_2, desc_2, ctx=ctx)
        fv.fp8_quantize_qkv_per_tensor(*dev, desc_2, *out_2, ctx=ctx)
        assert (_f32_bits(desc_f.cpu().numpy()) == _f32_bits(want)).all(), f
        r = ring_f.cpu().numpy()
        assert (_f32_bits(r[:48].reshape(3, 16)) == _f32_bits(ring_o.hist)).all(), f
        assert r[48:49].view(np.int32)[0] == ring_o.pos[0]
        assert torch.equal(ring_f, ring_2)
        for t in range(3):
            assert torch.equal(out_f[t], out_2[t]), (f, t)
        if f in (0, 16):  # spot-check the codes against the oracle quantizer
            for t in range(3):
                assert np.array_equal(_host_u8(out_f[t]),
                                      oracle.quantize_per_tensor(x[t], want[t]).reshape(-1)), (f, t)
    _check_ok(ctx)


@pytest.mark.parametrize("n", [0, 1, 7, 8, 9, 8 * 1000 + 5, 1 << 20, 3 * (1 << 22) + 3,
                               44 * (1 << 20) + 5])
def test_fused_amax_ring_quantize_ragged_sizes(ctx, n):
    """Ragged lengths (tails below one 16-byte vector, a grid larger than
    one block's share, inputs above twice L2, which take the two-kernel
    path): codes and descales equal the oracle's bit for bit."""
    bits = [np.ascontiguousarray(synth.bf16_tensor(synth.stream_key(n + 5, 1, t), 1, max(n, 1))[0, :n])
            for t in range(3)]
    if n:
        for t in range(3):
            bits[t][-1] = np.uint16(0xC2F0 + t)  # the largest magnitude sits in the tail
    ring_d = fv.new_ring()
    desc_d = torch.zeros(3, dtype=torch.float32, device="cuda")
    dev = [_dev_bf16(b) if n else torch.empty(8, dtype=torch.bfloat16, device="cuda") for b in bits]
    out = [torch.full((max(n, 8),), 0x7F, dtype=torch.uint8, device="cuda") for _ in range(3)]
    assert fv.lib().fp8_amax_ring_quantize_qkv(
        ctx.handle, dev[0].data_ptr(), dev[1].data_ptr(), dev[2].data_ptr(), n,
        ring_d.data_ptr(), desc_d.data_ptr(), out[0].data_ptr(), out[1].data_ptr(),
        out[2].data_ptr(), fv._stream()) == fv.OK
    _check_ok(ctx)
    want = oracle.Ring().update([oracle.amax_bf16(b) for b in bits])
    assert (_f32_bits(desc_d.cpu().numpy()) == _f32_bits(want)).all()
    for t in range(3):
        assert np.array_equal(_host_u8(out[t])[:n], oracle.quantize_per_tensor(bits[t], want[t]))


def test_fused_barrier_timeout_is_reported_and_recovered():
    """A lost arrival (injected on the host) makes the fused kernel's grid
    barrier wait run out: every block gives up after its bounded wait and
    returns, fp8vit_check reports FP8VIT_ETIMEOUT at site 200 and resets the
    reduction state, and the next call on the same context is bit-exact."""
    c = fv.Context()
    x = [synth.bf16_tensor(synth.stream_key(31, 0, t), 64, 1152) for t in range(3)]
    dev = [_dev_bf16(a).reshape(-1) for a in x]
    n = dev[0].numel()
    out = [torch.empty(n, dtype=torch.uint8, device="cuda") for _ in range(3)]
    ring_d = fv.new_ring()
    desc_d = torch.zeros(3, dtype=torch.float32, device="cuda")
    assert fv.lib().fp8vit_inject_lost_arrival(c.handle, fv._stream()) == fv.OK
    fv.fp8_amax_ring_quantize_qkv(*dev, ring_d, desc_d, *out, ctx=c)
    st, site = c.check()
    assert st == fv.ETIMEOUT and site == 200, (fv.status_string(st), site)
    assert c.check() == (fv.OK, 0)  # the fault was cleared
    ring_d = fv.new_ring()
    fv.fp8_amax_ring_quantize_qkv(*dev, ring_d, desc_d, *out, ctx=c)
    _check_ok(c)
    want = oracle.Ring().update([oracle.amax_bf16(a) for a in x])
    assert (_f32_bits(desc_d.cpu().numpy()) == _f32_bits(want)).all()
    for t in range(3):
        assert np.array_equal(_host_u8(out[t]), oracle.quantize_per_tensor(x[t], want[t]).reshape(-1))
    c.close()


@pytest.mark.parametrize("m,n", [(1, 2048), (1, 7168), (726, 7168), (1933, 7168), (37504, 2048)])
def test_group_quant_table_shapes(ctx, m, n):
    """Shapes of the per_token_group_quant_fp8 benchmark table (token_count x
    hidden_size): codes and scales equal the oracle's bit for bit."""
    x = synth.bf16_tensor(synth.stream_key(m, n, 0), m, n)
    xq = torch.empty((m, n), dtype=torch.uint8, device="cuda")
    sc = torch.empty((m, n // 128), dtype=torch.float32, device="cuda")
    fv.per_token_group_quant_fp8(_dev_bf16(x).reshape(m, n), 128, xq, sc, ctx=ctx)
    _check_ok(ctx)
    want_q, want_s = oracle.group_quant(x, 128)
    assert np.array_equal(_host_u8(xq), want_q)
    assert (_f32_bits(sc.cpu().numpy()) == _f32_bits(want_s)).all()
