"""The single-launch (streaming) prepass, sage_quant_qkv, at the workload
sizes, on its two K-mean paths, and its bounded waits.

Its outputs must equal those of the separate kernels (sage_quant_qk +
sage_quant_v) byte for byte, and the oracle's on sampled heads.  The K mean
is taken from an atomic FP64 accumulator for channels whose exponent range
makes every partial sum exact, and from the chunk partials in chunk order
otherwise (formed once per head by the K code tile that claims them); a
planted cancellation makes the chunk order matter, so only the second path
gives the oracle's value there.  Groups holding NaN, inf or
only tiny values take the reference form of the INT8 codes (conversion and
clamp) instead of the fast rounding; both forms are checked."""
import numpy as np
import pytest

import gpu_util as gu
import oracle
import synth

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def sage():
    import fp8_quantized_exact_b200 as s
    from fp8_quantized_exact_b200 import build
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()
    torch.cuda.set_device(torch.device("cuda:0"))
    return s


def _buffers(sage, B, N, H, D, dev, fill):
    shp = sage.quant_shapes(B, N, H, D)
    return {n: torch.full(s, fill, dtype=dt, device=dev) for (n, s), dt in zip(
        shp.items(), (torch.int8, torch.float32, torch.int8, torch.float32, torch.float32,
                      torch.uint8, torch.float32))}


def _qkv(sage, q, k, v, dev, fill=7):
    B, N, H, D = q.shape
    a = _buffers(sage, B, N, H, D, dev, fill)
    ws = sage.workspace(sage.SAGE_OP_QUANT_QKV, B, N, H, D, dev)
    sage.sage_quant_qkv(q, k, v, a["q_i8"], a["q_scale"], a["k_i8"], a["k_scale"], a["k_mean"],
                        a["v_fp8"], a["v_scale"], ws)
    return a, ws


def _separate(sage, q, k, v, dev):
    B, N, H, D = q.shape
    b = _buffers(sage, B, N, H, D, dev, 9)
    sage.sage_quant_qk(q, k, b["q_i8"], b["q_scale"], b["k_i8"], b["k_scale"], b["k_mean"],
                       sage.workspace(sage.SAGE_OP_QUANT_QK, B, N, H, D, dev))
    sage.sage_quant_v(v, b["v_fp8"], b["v_scale"], sage.workspace(sage.SAGE_OP_QUANT_V, B, N, H, D, dev))
    return b


def _logical(a, N, heads):
    """Oracle layout of the listed (b, h) heads, stacked as B=1."""
    get = {n: t.cpu().numpy() for n, t in a.items()}
    res = {"q8": get["q_i8"][:, :, :N], "q_scale": get["q_scale"], "k8": get["k_i8"][:, :, :N],
           "k_scale": get["k_scale"], "k_mean": get["k_mean"],
           "v8": get["v_fp8"][:, :, :, :N].transpose(0, 1, 3, 2), "v_scale": get["v_scale"]}
    return {n: np.stack([x[b, h] for b, h in heads])[None] for n, x in res.items()}


def _heads_view(x, heads):
    return np.ascontiguousarray(np.stack([x[b, :, h] for b, h in heads], axis=1)[None])


def _check_oracle(got, inp, heads, N):
    qz = oracle.quantize(_heads_view(inp.q, heads), _heads_view(inp.k, heads), _heads_view(inp.v, heads))
    for name in ("q8", "k8", "v8", "q_scale", "k_scale", "k_mean", "v_scale"):
        a, b = got[name], getattr(qz, name)
        assert a.shape == b.shape, name
        w = np.uint8 if a.dtype.itemsize == 1 else np.uint32
        bad = np.argwhere(a.view(w) != b.view(w))
        assert bad.size == 0, f"{name} differs at {bad[:4].tolist()}"


@pytest.mark.parametrize("cfg", ["outlier", "long_fused", "d64_batch"])
def test_single_launch_at_workload_sizes(sage, cfg):
    """The B2 N8192 H32, B1 N37810 H56 (fused projection strides) and B4
    N16384 H24 D64 workloads (the work list taken four tiles at a time): one
    launch, the separate kernels' bytes, and the oracle's bytes on three
    sampled heads."""
    dev = torch.device("cuda:0")
    c = synth.CONFIGS[cfg]
    assert sage.sage_quant_qkv_kernels(c.B, c.N, c.H, c.D) == 1
    inp = synth.make_inputs(c, seed=0)
    (q, k, v), _ = gu.to_device(inp, dev)
    a, ws = _qkv(sage, q, k, v, dev)
    assert sage.sage_read_device_status(ws) == sage.SAGE_OK
    b = _separate(sage, q, k, v, dev)
    torch.cuda.synchronize()
    for n in a:
        assert torch.equal(a[n].view(torch.uint8), b[n].view(torch.uint8)), n
    heads = [(0, 0), (c.B - 1, c.H // 2), (c.B - 1, c.H - 1)]
    _check_oracle(_logical(a, c.N, heads), inp, heads, c.N)


def test_chunk_order_path_for_channels_off_the_bound(sage):
    """Channel 5 of head 1: +2^30 and -2^30 in chunks 0 and 1, then 2^-30 in
    one token of each later chunk.  Added in chunk order the big values
    cancel first and every small one counts; in most other orders a small
    value meets an unbalanced 2^30 and is lost.  The channel fails the
    exactness bound, so the kernel must use the chunk-order sum.  Channel 9
    of head 0 holds one tiny value among normal ones (its chunk partial
    absorbs it).  All other channels take the accumulator path."""
    dev = torch.device("cuda:0")
    B, N, H, D = 1, 20 * 64 + 17, 3, 128
    inp = synth.custom(B, N, H, D, seed=77)
    kk = inp.k  # strided view into the generator's buffer: edits reach the bytes uploaded below

    def bf16(x):
        return np.float32(x).view(np.uint32) >> 16

    kk[0, :, 1, 5] = 0
    kk[0, 3, 1, 5] = bf16(2.0 ** 30)
    kk[0, 64 + 9, 1, 5] = bf16(-(2.0 ** 30))
    for c in range(2, 21):
        kk[0, 64 * c + (c % 17), 1, 5] = bf16(2.0 ** -30) if 64 * c + (c % 17) < N else 0
    kk[0, 200, 0, 9] = bf16(2.0 ** -100)
    assert sage.sage_quant_qkv_kernels(B, N, H, D) == 1
    (q, k, v), _ = gu.to_device(inp, dev)
    a, ws = _qkv(sage, q, k, v, dev)
    assert sage.sage_read_device_status(ws) == sage.SAGE_OK
    qz = oracle.quantize(inp.q, inp.k, inp.v)
    km = a["k_mean"].cpu().numpy()
    # the planted channel: chunk order keeps all 19 small values
    assert km[0, 1, 5] == np.float32(19 * 2.0 ** -30 / N), km[0, 1, 5]
    heads = [(0, h) for h in range(H)]
    _check_oracle(_logical(a, N, heads), inp, heads, N)
    b = _separate(sage, q, k, v, dev)
    for n in a:
        assert torch.equal(a[n].view(torch.uint8), b[n].view(torch.uint8)), n
    assert np.array_equal(km, qz.k_mean)


def test_chunk_order_path_with_the_list_taken_in_batches(sage):
    """The planted cancellation of the test above in two heads of a shape
    long enough that CTAs take the work list four tiles at a time (B1
    N46000 H4 D128: 14,400 tiles, at least 16 per CTA of a 148 x 6 grid).
    Both heads' channels fail the bound, so their first K code tiles claim
    the chunk-order sums and the head's other code tiles, on other CTAs,
    wait for them; a CTA keeps the means for its next tiles of the head."""
    dev = torch.device("cuda:0")
    B, N, H, D = 1, 46000, 4, 128
    inp = synth.custom(B, N, H, D, seed=91)
    kk = inp.k

    def bf16(x):
        return np.float32(x).view(np.uint32) >> 16

    T64 = -(-N // 64)
    for h, ch in ((1, 5), (3, 77)):
        kk[0, :, h, ch] = 0
        kk[0, 3, h, ch] = bf16(2.0 ** 30)
        kk[0, 64 + 9, h, ch] = bf16(-(2.0 ** 30))
        for c in range(2, T64):
            kk[0, 64 * c + (c % 17), h, ch] = bf16(2.0 ** -30) if 64 * c + (c % 17) < N else 0
    (q, k, v), _ = gu.to_device(inp, dev)
    a, ws = _qkv(sage, q, k, v, dev)
    assert sage.sage_read_device_status(ws) == sage.SAGE_OK
    km = a["k_mean"].cpu().numpy()
    n_small = sum(1 for c in range(2, T64) if 64 * c + (c % 17) < N)
    for h, ch in ((1, 5), (3, 77)):
        assert km[0, h, ch] == np.float32(n_small * 2.0 ** -30 / N), (h, km[0, h, ch])
    b = _separate(sage, q, k, v, dev)
    torch.cuda.synchronize()
    for n in a:
        assert torch.equal(a[n].view(torch.uint8), b[n].view(torch.uint8)), n
    heads = [(0, 1), (0, 3)]
    _check_oracle(_logical(a, N, heads), inp, heads, N)


def test_many_short_heads(sage):
    """B24 N100 H64 D64: 1,536 heads of two 64-token tiles each.  The list
    is taken four tiles at a time (15,360 tiles) and the lag is large (about
    180 heads between a head's statistics and its codes): the separate
    kernels' bytes, and the oracle's on two sampled heads."""
    dev = torch.device("cuda:0")
    B, N, H, D = 24, 100, 64, 64
    inp = synth.custom(B, N, H, D, seed=24)
    (q, k, v), _ = gu.to_device(inp, dev)
    a, ws = _qkv(sage, q, k, v, dev)
    assert sage.sage_read_device_status(ws) == sage.SAGE_OK
    b = _separate(sage, q, k, v, dev)
    torch.cuda.synchronize()
    for n in a:
        assert torch.equal(a[n].view(torch.uint8), b[n].view(torch.uint8)), n
    heads = [(0, 0), (B - 1, H - 1)]
    _check_oracle(_logical(a, N, heads), inp, heads, N)


def test_withheld_count_times_out_and_the_next_call_is_right(sage):
    """The first K statistics tile of head 2 is never counted in (the test
    hook): the waits of that head's K code tiles run out after about 1 ms,
    the status word says SAGE_ERR_TIMEOUT (wait site 45), the kernel
    returns, and the next call on the same context writes the separate
    kernels' bytes."""
    dev = torch.device("cuda:0")
    B, N, H, D = 1, 1000, 4, 128
    assert sage.sage_quant_qkv_kernels(B, N, H, D) == 1
    inp = synth.custom(B, N, H, D, seed=12)
    (q, k, v), _ = gu.to_device(inp, dev)
    try:
        sage.sage_debug_set_stall(2, 2_000_000)
        a, ws = _qkv(sage, q, k, v, dev)
        st = sage.sage_read_device_status(ws)
        code, where, block = ws[:12].view(torch.int32).tolist()
    finally:
        sage.sage_debug_set_stall(-1, 0)
    assert st == sage.SAGE_ERR_TIMEOUT and where == 45, (st, where, block)
    a, ws = _qkv(sage, q, k, v, dev)
    assert sage.sage_read_device_status(ws) == sage.SAGE_OK
    b = _separate(sage, q, k, v, dev)
    for n in a:
        assert torch.equal(a[n].view(torch.uint8), b[n].view(torch.uint8)), n


def _ref_codes(x, inv):
    """Reference form of the INT8 codes in numpy: RNE(fl32(x * inv)) clamped
    to +-127; a NaN product gives 0."""
    y = (x.astype(np.float32) * np.float32(inv)).astype(np.float32)
    r = np.rint(y)
    r = np.where(np.isnan(r), 0.0, np.clip(r, -127, 127))
    return r.astype(np.int8)


def test_non_finite_and_tiny_groups_take_the_reference_form(sage):
    """NaN and inf in some Q rows and K/V tokens, and a head whose Q and K
    values are all tiny (inv = 127/amax overflows): the single launch and
    the separate kernels write the same bytes, and Q codes of those groups
    equal the reference form."""
    dev = torch.device("cuda:0")
    B, N, H, D = 1, 700, 3, 128
    inp = synth.custom(B, N, H, D, seed=5)

    def bf16(x):
        return np.float32(x).view(np.uint32) >> 16

    inp.q[0, 40, 0, 3] = bf16(np.nan)
    inp.q[0, 100, 0, 7] = bf16(np.inf)
    inp.q[0, 101, 0, 9] = bf16(-np.inf)
    inp.k[0, 300, 0, 11] = bf16(np.inf)
    inp.v[0, 200, 0, 5] = bf16(np.nan)
    tiny = (synth.bf16_to_float(inp.q[0, :, 2]) * np.float32(1e-38)).astype(np.float32)
    inp.q[0, :, 2] = tiny.view(np.uint32) >> 16
    tinyk = (synth.bf16_to_float(inp.k[0, :, 2]) * np.float32(1e-38)).astype(np.float32)
    inp.k[0, :, 2] = tinyk.view(np.uint32) >> 16
    assert sage.sage_quant_qkv_kernels(B, N, H, D) == 1
    (q, k, v), _ = gu.to_device(inp, dev)
    a, ws = _qkv(sage, q, k, v, dev)
    assert sage.sage_read_device_status(ws) == sage.SAGE_OK
    b = _separate(sage, q, k, v, dev)
    torch.cuda.synchronize()
    for n in a:
        assert torch.equal(a[n].view(torch.uint8), b[n].view(torch.uint8)), n
    q8 = a["q_i8"].cpu().numpy()
    qs = a["q_scale"].cpu().numpy()
    qf = synth.bf16_to_float(inp.q)
    for h, g in ((0, 1), (0, 3), (2, 0), (2, 5)):
        x = qf[0, 32 * g:32 * g + 32, h]
        am = np.nanmax(np.abs(np.where(np.isnan(x), 0, x)))
        with np.errstate(invalid="ignore", over="ignore"):  # 127 / amax overflows for the tiny head
            inv = np.float32(127.0) / np.float32(am) if am > 0 else np.float32(0)
            want = _ref_codes(x, inv)
        got = q8[0, h, 32 * g:32 * g + 32]
        assert np.array_equal(got, want), (h, g)
        assert qs[0, h, g] == (np.float32(am) / np.float32(127.0) if am > 0 else 0), (h, g)


def test_long_heads_take_one_launch(sage):
    """N = 40,000 at D = 128 (625 chunks of 64 tokens per head, past what a
    scheme that keeps a head's slices on chip would hold): still one launch,
    the separate kernels' bytes, the oracle's on a sampled head, and a clean
    status."""
    dev = torch.device("cuda:0")
    B, N, H, D = 1, 40000, 2, 128
    assert sage.sage_quant_qkv_kernels(B, N, H, D) == 1
    inp = synth.custom(B, N, H, D, seed=40)
    (q, k, v), _ = gu.to_device(inp, dev)
    a, ws = _qkv(sage, q, k, v, dev)
    assert sage.sage_read_device_status(ws) == sage.SAGE_OK
    b = _separate(sage, q, k, v, dev)
    torch.cuda.synchronize()
    for n in a:
        assert torch.equal(a[n].view(torch.uint8), b[n].view(torch.uint8)), n
    heads = [(0, 1)]
    _check_oracle(_logical(a, N, heads), inp, heads, N)
