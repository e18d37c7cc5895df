"""Kernel-level parity: each CUDA entry point against the oracle's definition
of the same step, on seeded inputs that span several tiles and a ragged
tail.  Error bounds come from the arithmetic: f16 operands are exact in the
f32 products, so a K-term f32 accumulation is within K * 2^-22 * sum|a w| of
the exact sum; an f16 result adds one rounding of 2^-11 relative."""
import numpy as np
import pytest

from tests.gpu_common import dev, f16_values, host, need_cuda, orc, synth, torch

import jepa_video_encoder_b200 as jb

pytestmark = pytest.mark.gpu

U22 = 2.0 ** -22


def _ok():
    assert jb.op_sync_status() == 0


# ------------------------------------------------------------- LayerNorm ----
@pytest.mark.parametrize("rows,D", [(1000, 1024), (257, 192), (37, 4096), (1, 64)])
def test_layernorm(rows, D):
    need_cuda()
    rng = np.random.default_rng(rows + D)
    x = (rng.standard_normal((rows, D)) * 2 + 0.5).astype(np.float32)
    g = (1 + 0.1 * rng.standard_normal(D)).astype(np.float32)
    b = (0.05 * rng.standard_normal(D)).astype(np.float32)
    ref = orc.layer_norm(x.astype(np.float64), g.astype(np.float64), b.astype(np.float64), 1e-6)
    o32 = torch.empty((rows, D), dtype=torch.float32, device="cuda")
    o16 = torch.empty((rows, D), dtype=torch.float16, device="cuda")
    xd, gd, bd = dev(x), dev(g), dev(b)
    jb.layernorm(xd, gd, bd, 1e-6, o32)
    jb.layernorm(xd, gd, bd, 1e-6, o16)
    _ok()
    assert np.all(np.abs(host(o32) - ref) <= 2e-5 * (np.abs(ref) + 1))
    assert np.all(np.abs(host(o16) - ref) <= 2.0 ** -11 * np.abs(ref) + 3e-5 * (np.abs(ref) + 1))


def test_layernorm_strided_rows():
    """The CLS-pooling form: output row r normalises input row r * stride."""
    need_cuda()
    rng = np.random.default_rng(3)
    B, N, D = 3, 5, 256
    x = rng.standard_normal((B * N, D)).astype(np.float32)
    g = np.ones(D, np.float32)
    b = np.zeros(D, np.float32)
    out = torch.empty((B, D), dtype=torch.float32, device="cuda")
    jb.layernorm(dev(x), dev(g), dev(b), 1e-6, out, in_row_stride=N, rows=B)
    _ok()
    ref = orc.layer_norm(x[::N].astype(np.float64), 1.0, 0.0, 1e-6)
    assert np.allclose(host(out), ref, rtol=2e-5, atol=2e-5)


# ------------------------------------------------------------------ GEMM ----
def _gemm_inputs(M, K, N, seed):
    rng = np.random.default_rng(seed)
    A = rng.standard_normal((M, K)).astype(np.float16)
    W = (0.05 * rng.standard_normal((N, K))).astype(np.float16)
    bias = (0.1 * rng.standard_normal(N)).astype(np.float32)
    return A, W, bias


def _gemm_bound(A64, W64, K):
    return K * U22 * (np.abs(A64) @ np.abs(W64).T)


@pytest.mark.parametrize("M,K,N", [(300, 1024, 768), (1, 256, 576), (129, 192, 640), (2000, 512, 1024)])
def test_linear_f32_epilogue(M, K, N):
    need_cuda()
    A, W, bias = _gemm_inputs(M, K, N, M + N)
    A64, W64 = A.astype(np.float64), W.astype(np.float64)
    ref = A64 @ W64.T + bias
    out = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
    jb.linear(dev(A), dev(W), synth.DT_F16, N, dev(bias), jb._abi.EPI_F32, out)
    _ok()
    err = np.abs(host(out) - ref)
    assert np.all(err <= _gemm_bound(A64, W64, K) + U22 * np.abs(ref) + 1e-30)


@pytest.mark.parametrize("epi", ["f16", "gelu", "resid"])
def test_linear_epilogues(epi):
    need_cuda()
    M, K, N = 333, 1024, 1024
    A, W, bias = _gemm_inputs(M, K, N, 7)
    A64, W64 = A.astype(np.float64), W.astype(np.float64)
    ref = A64 @ W64.T + bias
    bnd = _gemm_bound(A64, W64, K) + U22 * np.abs(ref)
    if epi == "f16":
        out = torch.empty((M, N), dtype=torch.float16, device="cuda")
        jb.linear(dev(A), dev(W), synth.DT_F16, N, dev(bias), jb._abi.EPI_F16, out)
        _ok()
        assert np.all(np.abs(host(out) - ref) <= bnd + 2.0 ** -11 * np.abs(ref) + 1e-7)
    elif epi == "gelu":
        out = torch.empty((M, N), dtype=torch.float16, device="cuda")
        jb.linear(dev(A), dev(W), synth.DT_F16, N, dev(bias), jb._abi.EPI_GELU_F16, out)
        _ok()
        g = orc.gelu(ref)
        # |gelu'| <= 1.13; erff is within a few ulp of erf
        assert np.all(np.abs(host(out) - g) <= 1.13 * bnd + 2.0 ** -11 * np.abs(g) + 1e-6)
    else:
        base = np.random.default_rng(8).standard_normal((M, N)).astype(np.float32)
        out = dev(base)
        jb.linear(dev(A), dev(W), synth.DT_F16, N, dev(bias), jb._abi.EPI_RESID_F32, out)
        _ok()
        want = base.astype(np.float64) + ref
        assert np.all(np.abs(host(out) - want) <= bnd + U22 * np.abs(want) + 1e-30)


def _quant_weight(wdt, N, K, seed):
    rng = np.random.default_rng(seed)
    W = (0.05 * rng.standard_normal((N, K))).astype(np.float32)
    blocks = synth.quantize_q8_0(W) if wdt == "q8_0" else synth.quantize_q4_0(W)
    deq = (orc.dequant_q8_0 if wdt == "q8_0" else orc.dequant_q4_0)(blocks, N * K).reshape(N, K)
    dt = synth.DTYPE_IDS[wdt]
    qs = torch.empty((N, K if wdt == "q8_0" else K // 2), dtype=torch.uint8, device="cuda")
    sc = torch.empty((N, K // 32), dtype=torch.float16, device="cuda")
    jb.repack(dt, dev(blocks), N, K, qs, sc)
    return dt, blocks, deq, qs, sc


@pytest.mark.parametrize("wdt", ["q8_0", "q4_0"])
def test_quant_unpack_bit_exact(wdt):
    """A = identity makes the GEMM output the weight operand itself: every
    unpacked value equals binary16(q*d) / binary16((q-8)*d) of the oracle's
    dequantisation exactly, over all codes and random scales.  (Values are
    compared, not bit patterns: the GEMM sums 1*w with zero products, which
    turns a -0.0 weight into +0.0.)"""
    need_cuda()
    N, K = 512, 256
    dt, blocks, deq, qs, sc = _quant_weight(wdt, N, K, 11)
    # every code appears: q8 [-127, 127], q4 [0, 15]
    eye = np.eye(K, dtype=np.float16)
    out = torch.empty((K, N), dtype=torch.float32, device="cuda")
    jb.linear(dev(eye), qs, dt, N, None, jb._abi.EPI_F32, out, w_scales=sc)
    _ok()
    got = out.cpu().numpy()
    want = f16_values(deq).T.astype(np.float32)
    assert np.array_equal(got, want)
    # the repack kernel moved bytes only
    bs = 34 if wdt == "q8_0" else 18
    raw = blocks.reshape(-1, bs)
    assert np.array_equal(sc.cpu().numpy().view(np.uint8).reshape(-1, 2), raw[:, :2])
    assert np.array_equal(qs.cpu().numpy().reshape(-1, bs - 2), raw[:, 2:])


@pytest.mark.parametrize("wdt", ["q8_0", "q4_0"])
def test_dequant_f16_bit_exact(wdt):
    """The f16 copy the large-M GEMMs use holds binary16(q*d) / binary16((q-8)*d)
    of the oracle's dequantisation, bit for bit, over all codes."""
    need_cuda()
    N, K = 384, 512
    dt, blocks, deq, qs, sc = _quant_weight(wdt, N, K, 13)
    out = torch.empty((N, K), dtype=torch.float16, device="cuda")
    jb.dequant_f16(dt, qs, sc, N, K, out)
    _ok()
    want = deq.astype(np.float16)  # one rounding of the exact product (q*d is exact in float64)
    assert np.array_equal(out.cpu().numpy().view(np.uint16), want.view(np.uint16))


@pytest.mark.parametrize("wdt", ["q8_0", "q4_0"])
@pytest.mark.parametrize("M,K,N", [(300, 1024, 768), (1000, 4096, 1024)])
def test_linear_quant(wdt, M, K, N):
    need_cuda()
    dt, blocks, deq, qs, sc = _quant_weight(wdt, N, K, M)
    rng = np.random.default_rng(5)
    A = rng.standard_normal((M, K)).astype(np.float16)
    bias = (0.1 * rng.standard_normal(N)).astype(np.float32)
    out = torch.empty((M, N), dtype=torch.float32, device="cuda")
    jb.linear(dev(A), qs, dt, N, dev(bias), jb._abi.EPI_F32, out, w_scales=sc)
    _ok()
    A64 = A.astype(np.float64)
    Wop = f16_values(deq)
    ref = A64 @ Wop.T + bias
    assert np.all(np.abs(host(out) - ref) <= _gemm_bound(A64, Wop, K) + U22 * np.abs(ref) + 1e-30)
    # and against the exact dequantised weights (the f16 operand rounding)
    exact = A64 @ deq.T + bias
    cos = orc.token_cosines(host(out), exact)
    assert cos.min() > 0.99999


def test_linear_full_qkv_shape_sampled():
    """The LeVJEPA ViT-L QKV shape at batch 4 (12548 x 1024 x 3072): 1188
    output tiles through the persistent scheduler, sampled rows checked."""
    need_cuda()
    M, K, N = 4 * 3137, 1024, 3072
    A, W, bias = _gemm_inputs(M, K, N, 21)
    out = torch.empty((M, N), dtype=torch.float32, device="cuda")
    jb.linear(dev(A), dev(W), synth.DT_F16, N, dev(bias), jb._abi.EPI_F32, out)
    _ok()
    rows = np.r_[0:3, 127:130, 6000:6003, M - 3:M]
    A64, W64 = A[rows].astype(np.float64), W.astype(np.float64)
    ref = A64 @ W64.T + bias
    got = host(out[torch.as_tensor(rows).cuda()])
    assert np.all(np.abs(got - ref) <= _gemm_bound(A64, W64, K) + U22 * np.abs(ref) + 1e-30)


@pytest.mark.parametrize("first_part,parts", [(0, 3), (1, 2)])
def test_qkv_scatter(first_part, parts):
    need_cuda()
    B, ntok, heads = 3, 130, 2
    D = 64 * heads
    K, N = 256, parts * D
    npad = 256
    A, W, bias = _gemm_inputs(B * ntok, K, N, 31 + parts)
    q = torch.zeros((B * heads, ntok, 64), dtype=torch.float16, device="cuda")
    k = torch.zeros_like(q)
    vt = torch.zeros((B * heads, 64, npad), dtype=torch.float16, device="cuda")
    jb.linear_qkv(dev(A), dev(W), synth.DT_F16, N, dev(bias), ntok, heads, npad, first_part,
                  q if first_part == 0 else None, k, vt)
    _ok()
    ref = A.astype(np.float64) @ W.astype(np.float64).T + bias
    bnd = _gemm_bound(A.astype(np.float64), W.astype(np.float64), K) + 2.0 ** -11 * np.abs(ref) + 1e-7
    names = ["q", "k", "v"][first_part:]
    for pi, name in enumerate(names):
        part = ref[:, pi * D:(pi + 1) * D].reshape(B, ntok, heads, 64).transpose(0, 2, 1, 3)
        pb = bnd[:, pi * D:(pi + 1) * D].reshape(B, ntok, heads, 64).transpose(0, 2, 1, 3)
        if name == "v":
            got = host(vt).reshape(B, heads, 64, npad)
            assert np.all(got[..., ntok:] == 0)
            got = got[..., :ntok].transpose(0, 1, 3, 2)
        else:
            got = host(q if name == "q" else k).reshape(B, heads, ntok, 64)
        assert np.all(np.abs(got - part) <= pb), name


# ------------------------------------------------------------- attention ----
def _attn_case(B, heads, n_patches, ppf, has_cls, mask, seed, qscale=3.0):
    rng = np.random.default_rng(seed)
    N = n_patches + (1 if has_cls else 0)
    npad = (N + 127) // 128 * 128
    q = (qscale * rng.standard_normal((B * heads, N, 64))).astype(np.float16)
    k = rng.standard_normal((B * heads, N, 64)).astype(np.float16)
    v = rng.standard_normal((B * heads, N, 64)).astype(np.float16)
    vt = np.zeros((B * heads, 64, npad), np.float16)
    vt[:, :, :N] = v.transpose(0, 2, 1)
    out = torch.full((B * N, heads * 64), float("nan"), dtype=torch.float16, device="cuda")
    jb.attention(dev(q), dev(k), dev(vt), B, heads, N, npad, synth.MASK_IDS[mask], int(has_cls), ppf, out)
    _ok()
    allow = None if mask == "bidir" else orc.allowed_keys(n_patches, ppf, has_cls, mask)
    return q, k, v, allow, host(out).reshape(B, N, heads, 64).transpose(0, 2, 1, 3).reshape(B * heads, N, 64)


@pytest.mark.parametrize("B,heads,n_patches,ppf,has_cls,mask", [
    (2, 2, 299, 23, True, "block_causal"),     # 300 tokens: 3 query tiles, ragged
    (1, 3, 256, 256, True, "bidir"),           # LeWM shape: 257 tokens
    (2, 1, 260, 4, False, "block_causal"),     # tiny slots: rows see keys in few tiles
    (1, 2, 64 * 4, 4, True, "block_causal"),   # slots of 4 with CLS
    (2, 2, 384, 96, True, "block_causal"),     # 385 tokens: 4 query tiles, the CLS row in a CTA of its own
    (1, 1, 127, 127, True, "block_causal"),    # 128 tokens: one query tile, paired with the CLS tile
    (1, 1, 1000, 1000, False, "bidir"),
])
def test_attention(B, heads, n_patches, ppf, has_cls, mask):
    need_cuda()
    q, k, v, allow, got = _attn_case(B, heads, n_patches, ppf, has_cls, mask, n_patches + heads)
    ref = orc.attention(q.astype(np.float64), k.astype(np.float64), v.astype(np.float64), allow)
    assert np.isfinite(got).all()
    assert np.abs(got - ref).max() <= 5e-3
    assert orc.token_cosines(got, ref).min() >= 0.9999


@pytest.mark.parametrize("n_patches,ppf,has_cls,mask,B", [
    (16 * 196, 196, True, "block_causal", 4),   # LeVJEPA ViT-L/16, 16 frames at 224^2
    (32 * 256, 256, False, "bidir", 2),         # V-JEPA 2 64-frame clip
])
def test_attention_full_size_sampled(n_patches, ppf, has_cls, mask, B):
    need_cuda()
    heads = 16
    q, k, v, allow, got = _attn_case(B, heads, n_patches, ppf, has_cls, mask, 99)
    N = q.shape[1]
    rows = np.unique(np.r_[0, 1, 2, 127, 128, 195, 196, 197, N // 2, N - 130, N - 2, N - 1])
    for bh in (0, B * heads // 2 + 3, B * heads - 1):
        ref = orc.attention(q[bh, rows].astype(np.float64), k[bh].astype(np.float64),
                            v[bh].astype(np.float64), None if allow is None else allow[rows])
        assert np.abs(got[bh, rows] - ref).max() <= 5e-3
        assert orc.token_cosines(got[bh, rows], ref).min() >= 0.9999


def test_attention_block_causal_perturbation_bit_identical():
    """Changing the keys / values of slot t+1 leaves the outputs of rows in
    slots <= t bit-identical (masked keys contribute exact zeros)."""
    need_cuda()
    B, heads, ppf, T = 1, 2, 50, 6
    n_patches = ppf * T
    N = n_patches + 1
    npad = (N + 127) // 128 * 128
    rng = np.random.default_rng(4)
    q = rng.standard_normal((B * heads, N, 64)).astype(np.float16)
    k = rng.standard_normal((B * heads, N, 64)).astype(np.float16)
    v = rng.standard_normal((B * heads, N, 64)).astype(np.float16)

    def run(k, v):
        vt = np.zeros((B * heads, 64, npad), np.float16)
        vt[:, :, :N] = v.transpose(0, 2, 1)
        out = torch.empty((B * N, heads * 64), dtype=torch.float16, device="cuda")
        jb.attention(dev(q), dev(k), dev(vt), B, heads, N, npad, 1, 1, ppf, out)
        _ok()
        return out.cpu().numpy()

    base = run(k, v)
    t = 2
    sl = slice(1 + (t + 1) * ppf, 1 + (t + 2) * ppf)
    k2, v2 = k.copy(), v.copy()
    k2[:, sl] = rng.standard_normal(k2[:, sl].shape)
    v2[:, sl] = rng.standard_normal(v2[:, sl].shape)
    new = run(k2, v2)
    keep = 1 + (t + 1) * ppf
    assert np.array_equal(new[1:keep].view(np.uint16), base[1:keep].view(np.uint16))
    assert not np.array_equal(new[keep:], base[keep:])
    assert not np.array_equal(new[0], base[0])


# ----------------------------------------------------------- patch-embed ----
@pytest.mark.parametrize("B,T,H,W,p,kt,D,has_cls", [
    (2, 4, 64, 48, 16, 2, 256, False),
    (1, 1, 224, 224, 14, 1, 192, True),        # LeWM: K = 588, padded to 640
    (3, 3, 32, 32, 16, 1, 128, True),
    # the general gather (patch rows not a multiple of 8 pixels): tubelet 2,
    # ragged K blocks, a ragged row tile, several row tiles
    (2, 4, 36, 60, 12, 2, 128, False),
    (3, 2, 42, 28, 14, 2, 192, True),
    (2, 2, 112, 98, 14, 1, 128, True),
])
def test_patch_embed(B, T, H, W, p, kt, D, has_cls):
    need_cuda()
    rng = np.random.default_rng(B * T + p)
    pix = rng.standard_normal((B, T, 3, H, W)).astype(np.float32)
    w = (0.02 * rng.standard_normal((D, 3, kt, p, p))).astype(np.float16)
    bias = (0.02 * rng.standard_normal(D)).astype(np.float32)
    n_patches = (T // kt) * (H // p) * (W // p)
    ntok = n_patches + (1 if has_cls else 0)
    pos = (0.02 * rng.standard_normal((ntok, D))).astype(np.float32)
    cls = (0.02 * rng.standard_normal(D)).astype(np.float32)
    K = 3 * kt * p * p
    kpad = (K + 63) // 64 * 64
    wpad = np.zeros((D, kpad), np.float16)
    wpad[:, :K] = w.reshape(D, K)
    x = torch.full((B, ntok, D), float("nan"), dtype=torch.float32, device="cuda")
    jb.patch_embed(dev(pix), p, kt, dev(wpad), D, dev(bias), dev(pos), dev(cls) if has_cls else None,
                   int(has_cls), x)
    _ok()
    got = host(x)

    def ref_with(pixels):
        e = orc.patch_embed(pixels, w.astype(np.float64), bias.astype(np.float64), p, kt)
        if has_cls:
            e = np.concatenate([np.broadcast_to(cls.astype(np.float64), (B, 1, D)), e], 1)
        return e + pos

    # with the f16-rounded pixels the GEMM is exact up to the f32 accumulation
    ref16 = ref_with(f16_values(pix))
    cols = orc.patchify(f16_values(pix), p, kt)
    bnd = K * U22 * (np.abs(cols) @ np.abs(w.reshape(D, K).astype(np.float64)).T)
    if has_cls:
        bnd = np.concatenate([np.zeros((B, 1, D)), bnd], 1)
    assert np.all(np.abs(got - ref16) <= bnd + U22 * (np.abs(ref16) + 1))
    assert orc.token_cosines(got, ref_with(pix.astype(np.float64))).min() >= 0.9999


# ----------------------------------------------------- head small kernels ----
@pytest.mark.parametrize("wdt", ["f16", "q8_0", "q4_0"])
@pytest.mark.parametrize("epi", [0, 1, 2])
def test_gemv(wdt, epi):
    need_cuda()
    M, K, N = 5, 1024, 174
    rng = np.random.default_rng(epi + 10)
    x = rng.standard_normal((M, K)).astype(np.float32)
    bias = (0.1 * rng.standard_normal(N)).astype(np.float32)
    if wdt == "f16":
        W16 = (0.05 * rng.standard_normal((N, K))).astype(np.float16)
        Wv, wd, sc, dt = W16.astype(np.float64), dev(W16), None, synth.DT_F16
    else:
        dt, blocks, Wv, wd, sc = _quant_weight(wdt, N, K, 3)
    resid = rng.standard_normal((M, N)).astype(np.float32)
    y = dev(resid) if epi == 2 else torch.empty((M, N), dtype=torch.float32, device="cuda")
    jb.gemv(dev(x), wd, dt, N, dev(bias), epi, y, resid=y if epi == 2 else None, resid_row_stride=N,
            w_scales=sc)
    _ok()
    lin = x.astype(np.float64) @ Wv.T + bias
    bnd = K * U22 * (np.abs(x.astype(np.float64)) @ np.abs(Wv).T) + U22 * np.abs(lin) + 1e-7
    want = {0: lin, 1: orc.gelu(lin), 2: resid + lin}[epi]
    assert np.all(np.abs(host(y) - want) <= 1.13 * bnd + 1e-6 * np.abs(want) + 1e-7)


def test_xattn_1q():
    need_cuda()
    B, heads, N = 3, 4, 2048
    npad = 2048
    rng = np.random.default_rng(12)
    q = (2 * rng.standard_normal(heads * 64)).astype(np.float32)
    k = rng.standard_normal((B * heads, N, 64)).astype(np.float16)
    v = rng.standard_normal((B * heads, N, 64)).astype(np.float16)
    vt = np.ascontiguousarray(v.transpose(0, 2, 1))
    out = torch.empty((B, heads * 64), dtype=torch.float32, device="cuda")
    jb.xattn_1q(dev(q), dev(k), dev(vt), B, heads, N, npad, out)
    _ok()
    qh = np.broadcast_to(q.reshape(1, heads, 1, 64), (B, heads, 1, 64)).astype(np.float64)
    ref = orc.attention(qh, k.reshape(B, heads, N, 64).astype(np.float64),
                        v.reshape(B, heads, N, 64).astype(np.float64), None).reshape(B, heads * 64)
    assert np.abs(host(out) - ref).max() <= 2e-5


def test_mean_pool():
    need_cuda()
    B, N, D = 3, 3137, 1024
    y = np.random.default_rng(13).standard_normal((B, N, D)).astype(np.float32)
    out = torch.empty((B, D), dtype=torch.float32, device="cuda")
    jb.mean_pool(dev(y), B, N, D, 1, out)
    _ok()
    ref = y[:, 1:].astype(np.float64).mean(1)
    assert np.abs(host(out) - ref).max() <= 1e-5


# ------------------------------------------------------------- timeouts ----
def test_bounded_wait_timeout_reports_and_recovers():
    """A zero wait bound makes the GEMM's first unfinished wait give up: the
    kernel unwinds (no trap), the status comes back as ERR_TIMEOUT, and the
    context stays usable for the next correct call."""
    need_cuda()
    M, K, N = 256, 1024, 512
    A, W, bias = _gemm_inputs(M, K, N, 41)
    out = torch.empty((M, N), dtype=torch.float32, device="cuda")
    jb.op_set_timeout_ns(0)
    try:
        jb.linear(dev(A), dev(W), synth.DT_F16, N, dev(bias), jb._abi.EPI_F32, out)
        st = jb.op_sync_status()
    finally:
        jb.op_set_timeout_ns(4_000_000_000)
    assert st == jb._abi.ERR_TIMEOUT
    jb.linear(dev(A), dev(W), synth.DT_F16, N, dev(bias), jb._abi.EPI_F32, out)
    _ok()
    ref = A.astype(np.float64) @ W.astype(np.float64).T + bias
    assert np.allclose(host(out), ref, rtol=1e-4, atol=1e-4)
