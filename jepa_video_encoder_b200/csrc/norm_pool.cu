// Memory-bound kernels of the encoder forward: the fused LayerNorm (pre-LN
// block norms, the final `norm`, the head's ln_kv / ln2), the CLS rows of the
// embedding, mean pooling over the patch tokens, and the byte repack of
// q8_0 / q4_0 blocks into the GEMM's layout.
//
// LayerNorm: y = (x - mean) / sqrt(var + eps) * gamma + beta over each row,
// biased variance, statistics in f32 from a row held in registers (two
// passes over registers, one pass over HBM).  One warp per row.
#include <algorithm>

#include "internal.h"
#include "patchify.h"

namespace jb {

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Output row r reads input row (r / grp) * grp_stride + grp_off + r % grp:
// consecutive rows (grp >= rows, grp_stride 0, grp_off 0), every in_stride-th
// row (grp 1, grp_stride in_stride), or a block of grp rows at offset grp_off
// in every group of grp_stride rows.
struct RowMap {
  int grp;
  long long grp_stride;
  int grp_off;
};

template <int MAXV, bool OUT_F16, bool BF>
__global__ void __launch_bounds__(256) layernorm_kernel(const float* __restrict__ x, int rows, int D, RowMap map,
                                                       const float* __restrict__ g, const float* __restrict__ b,
                                                       float eps, void* out) {
  pdl_wait();
  pdl_trigger();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nv = D >> 2;
  // grid-stride over rows: the grid is sized to the resident capacity
  for (int row = blockIdx.x * 8 + warp; row < rows; row += gridDim.x * 8) {
    const int gi = row / map.grp;
    const long long in_row = gi * map.grp_stride + map.grp_off + (row - gi * map.grp);
    const float4* xr = reinterpret_cast<const float4*>(x + static_cast<size_t>(in_row) * D);
    float4 v[MAXV];
    float s = 0.0f;
#pragma unroll
    for (int i = 0; i < MAXV; ++i) {
      const int idx = lane + 32 * i;
      if (idx < nv) {
        v[i] = __ldg(xr + idx);
        s += (v[i].x + v[i].y) + (v[i].z + v[i].w);
      } else {
        v[i] = make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
    const float mean = warp_sum(s) / static_cast<float>(D);
    float q = 0.0f;
#pragma unroll
    for (int i = 0; i < MAXV; ++i) {
      if (lane + 32 * i < nv) {
        const float a = v[i].x - mean, bb = v[i].y - mean, c = v[i].z - mean, d = v[i].w - mean;
        q += (a * a + bb * bb) + (c * c + d * d);
      }
    }
    const float rstd = rsqrtf(warp_sum(q) / static_cast<float>(D) + eps);
    const float4* g4 = reinterpret_cast<const float4*>(g);
    const float4* b4 = reinterpret_cast<const float4*>(b);
#pragma unroll
    for (int i = 0; i < MAXV; ++i) {
      const int idx = lane + 32 * i;
      if (idx < nv) {
        const float4 gg = __ldg(g4 + idx), bb = __ldg(b4 + idx);
        const float y0 = (v[i].x - mean) * rstd * gg.x + bb.x;
        const float y1 = (v[i].y - mean) * rstd * gg.y + bb.y;
        const float y2 = (v[i].z - mean) * rstd * gg.z + bb.z;
        const float y3 = (v[i].w - mean) * rstd * gg.w + bb.w;
        if (OUT_F16) {
          uint2* o = reinterpret_cast<uint2*>(static_cast<__half*>(out) + static_cast<size_t>(row) * D) + idx;
          *o = make_uint2(pack2<BF>(y0, y1), pack2<BF>(y2, y3));
        } else {
          float4* o = reinterpret_cast<float4*>(static_cast<float*>(out) + static_cast<size_t>(row) * D) + idx;
          *o = make_float4(y0, y1, y2, y3);
        }
      }
    }
  }
}

template <bool BF>
static void launch_ln(const float* x, int rows, int D, RowMap map, const float* g, const float* b, float eps,
                      void* out, bool out16, cudaStream_t st) {
  const dim3 grid(std::min((rows + 7) / 8, num_sms() * 8));
  if (D <= 1024) {
    if (out16)
      launch_pdl(layernorm_kernel<8, true, BF>, grid, dim3(256), 0, st, 1, x, rows, D, map, g, b, eps, out);
    else
      launch_pdl(layernorm_kernel<8, false, BF>, grid, dim3(256), 0, st, 1, x, rows, D, map, g, b, eps, out);
  } else {
    if (out16)
      launch_pdl(layernorm_kernel<32, true, BF>, grid, dim3(256), 0, st, 1, x, rows, D, map, g, b, eps, out);
    else
      launch_pdl(layernorm_kernel<32, false, BF>, grid, dim3(256), 0, st, 1, x, rows, D, map, g, b, eps, out);
  }
}

int launch_layernorm_rows(const float* x, int rows, int D, int grp, long long grp_stride, int grp_off, const float* g,
                          const float* b, float eps, void* out, bool out_f16, cudaStream_t st, bool bf16) {
  if (!x || !g || !b || !out) return JEPA_B200_ERR_ARG;
  if (rows < 1 || D < 4 || D % 4 != 0 || D > 4096 || grp < 1 || grp_stride < 0 || grp_off < 0)
    return JEPA_B200_ERR_SHAPE;
  const RowMap map{grp, grp_stride, grp_off};
  if (bf16)
    launch_ln<true>(x, rows, D, map, g, b, eps, out, out_f16, st);
  else
    launch_ln<false>(x, rows, D, map, g, b, eps, out, out_f16, st);
  return cudaGetLastError() == cudaSuccess ? JEPA_B200_OK : JEPA_B200_ERR_CUDA;
}

int launch_layernorm(const float* x, int rows, int D, long long in_stride, const float* g, const float* b,
                     float eps, void* out, bool out_f16, cudaStream_t st, bool bf16) {
  if (in_stride < 1) return JEPA_B200_ERR_SHAPE;
  return in_stride == 1 ? launch_layernorm_rows(x, rows, D, rows, 0, 0, g, b, eps, out, out_f16, st, bf16)
                        : launch_layernorm_rows(x, rows, D, 1, in_stride, 0, g, b, eps, out, out_f16, st, bf16);
}

// x[b, 0, :] = cls + pos[0]
__global__ void cls_rows_kernel(float* x, int B, int ntok, int D, const float* cls, const float* pos) {
  pdl_wait();
  pdl_trigger();
  const int b = blockIdx.y;
  for (int c = blockIdx.x * blockDim.x + threadIdx.x; c < D; c += gridDim.x * blockDim.x)
    x[static_cast<size_t>(b) * ntok * D + c] = cls[c] + pos[c];
}

int launch_cls_rows(float* x, int B, int ntok, int D, const float* cls, const float* pos, cudaStream_t st) {
  if (!x || !cls || !pos) return JEPA_B200_ERR_ARG;
  launch_pdl(cls_rows_kernel, dim3((D + 255) / 256, B), dim3(256), 0, st, 1, x, B, ntok, D, cls, pos);
  return cudaGetLastError() == cudaSuccess ? JEPA_B200_OK : JEPA_B200_ERR_CUDA;
}

// Patch-embed, input side: the unfolded patch matrix of the tubelet
// convolution, rounded to the 16-bit type, as the A operand of a TMA-fed
// GEMM.  Row m = patch (clip b, slot t', patch row py, patch column px),
// column k = (c, dt, kh, kw) in the row-major order of a conv weight
// [D, 3, kt, p, p]; columns k >= 3 kt p^2 (up to the padded K) are zero.
// One thread writes 8 consecutive columns of one row (16 bytes); with
// p % 8 == 0 those are 8 consecutive pixels of one image row, read as two
// 16-byte loads when the image rows allow it.
template <bool BF>
__global__ void __launch_bounds__(256) patchify_kernel(const float* __restrict__ px, int T, int H, int W, int p,
                                                        int kt, int n_patches, long long rows, int K, int Kpad,
                                                        int vec, uint16_t* __restrict__ a) {
  pdl_wait();
  pdl_trigger();
  const int groups = Kpad / 8;
  const long long g = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (g >= rows * groups) return;
  const long long m = g / groups;
  const int k0 = static_cast<int>(g - m * groups) * 8;
  const long long b = m / n_patches;
  const int i = static_cast<int>(m - b * n_patches);
  const int wp = W / p, ppf = (H / p) * wp;
  const int ts = i / ppf, py = (i % ppf) / wp, pxi = i % wp;
  const size_t hw = static_cast<size_t>(H) * W;
  float v[8];
  if (vec && k0 + 8 <= K) {
    // 8 pixels of one image row (p % 8 == 0): kw = k0 % p .. + 7, 16-byte aligned
    const int kw = k0 % p, kh = (k0 / p) % p, dt = (k0 / (p * p)) % kt, c = k0 / (p * p * kt);
    const size_t f = static_cast<size_t>(b) * T + static_cast<size_t>(ts) * kt + dt;
    const float* src = px + (f * 3 + c) * hw + static_cast<size_t>(py * p + kh) * W + pxi * p + kw;
    const float4 u = __ldg(reinterpret_cast<const float4*>(src)), w = __ldg(reinterpret_cast<const float4*>(src + 4));
    v[0] = u.x;
    v[1] = u.y;
    v[2] = u.z;
    v[3] = u.w;
    v[4] = w.x;
    v[5] = w.y;
    v[6] = w.z;
    v[7] = w.w;
  } else {
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int k = k0 + e;
      v[e] = 0.0f;
      if (k < K) {
        const int kw = k % p, kh = (k / p) % p, dt = (k / (p * p)) % kt, c = k / (p * p * kt);
        const size_t f = static_cast<size_t>(b) * T + static_cast<size_t>(ts) * kt + dt;
        v[e] = __ldg(px + (f * 3 + c) * hw + static_cast<size_t>(py * p + kh) * W + pxi * p + kw);
      }
    }
  }
  *reinterpret_cast<uint4*>(a + m * Kpad + k0) =
      make_uint4(pack2<BF>(v[0], v[1]), pack2<BF>(v[2], v[3]), pack2<BF>(v[4], v[5]), pack2<BF>(v[6], v[7]));
}

int launch_patchify(const float* pixels, const PatchSrc& s, int B, int Kpad, void* a, cudaStream_t st, bool bf16) {
  if (!pixels || !a || B < 1) return JEPA_B200_ERR_ARG;
  if (Kpad % 8 != 0 || Kpad < s.k_real || s.patch < 1 || s.tubelet < 1 || (reinterpret_cast<uintptr_t>(a) & 15))
    return JEPA_B200_ERR_SHAPE;
  // 16-byte pixel loads need 8-pixel patch rows on 16-byte-aligned image rows
  const int vec = (s.patch % 8 == 0) && (s.W % 4 == 0) && ((static_cast<size_t>(s.H) * s.W) % 4 == 0) &&
                          ((reinterpret_cast<uintptr_t>(pixels) & 15) == 0)
                      ? 1
                      : 0;
  const long long rows = static_cast<long long>(B) * s.n_patches;
  const long long threads = rows * (Kpad / 8);
  launch_pdl(bf16 ? patchify_kernel<true> : patchify_kernel<false>, dim3(static_cast<unsigned>((threads + 255) / 256)),
             dim3(256), 0, st, 1, pixels, s.T, s.H, s.W, s.patch, s.tubelet, s.n_patches, rows, s.k_real, Kpad, vec,
             static_cast<uint16_t*>(a));
  return cudaGetLastError() == cudaSuccess ? JEPA_B200_OK : JEPA_B200_ERR_CUDA;
}

// Masked predictor, input side: the context rows of the encoder output
// gathered and rounded to f16 (the A operand of pred.embed), and the
// predictor's sequence [context | targets] of every clip assembled in f32.
// One CTA per output row.
// a[b * nsel + i, :] = f16(tokens[b, idx[i], :]); 8 columns per thread.
template <bool BF>
__global__ void gather_rows_f16_kernel(const float* __restrict__ tokens, const int* __restrict__ idx, int ntok,
                                       int nsel, int D, __half* __restrict__ a) {
  pdl_wait();
  pdl_trigger();
  const long long r = blockIdx.x;  // b * nsel + i
  const long long b = r / nsel;
  const int i = static_cast<int>(r - b * nsel);
  const float* src = tokens + (b * ntok + idx[i]) * D;
  __half* dst = a + r * D;
  for (int c = threadIdx.x * 8; c < D; c += blockDim.x * 8) {
    const float4 u = *reinterpret_cast<const float4*>(src + c), v = *reinterpret_cast<const float4*>(src + c + 4);
    *reinterpret_cast<uint4*>(dst + c) =
        make_uint4(pack2<BF>(u.x, u.y), pack2<BF>(u.z, u.w), pack2<BF>(v.x, v.y), pack2<BF>(v.z, v.w));
  }
}

int launch_gather_rows_f16(const float* tokens, const int* idx, int B, int ntok, int nsel, int D, __half* a,
                           cudaStream_t st, bool bf16) {
  if (!tokens || !idx || !a) return JEPA_B200_ERR_ARG;
  if (B < 1 || nsel < 1 || ntok < 1 || D < 8 || D % 8 != 0) return JEPA_B200_ERR_SHAPE;
  launch_pdl(bf16 ? gather_rows_f16_kernel<true> : gather_rows_f16_kernel<false>,
             dim3(static_cast<unsigned>(B) * nsel), dim3(128), 0, st, 1, tokens, idx, ntok, nsel, D, a);
  return cudaGetLastError() == cudaSuccess ? JEPA_B200_OK : JEPA_B200_ERR_CUDA;
}

// x[b, i, :] = e[b * nctx + i, :] + pos[ctx[i], :]            (i < nctx)
// x[b, nctx + t, :] = mask[:] + pos[tgt[t], :]                 (t < ntgt)
__global__ void pred_assemble_kernel(const float* __restrict__ e, const float* __restrict__ mask,
                                     const float* __restrict__ pos, const int* __restrict__ ctx,
                                     const int* __restrict__ tgt, int nctx, int ntgt, int D, float* __restrict__ x) {
  pdl_wait();
  pdl_trigger();
  const int L = nctx + ntgt;
  const long long r = blockIdx.x;  // b * L + j
  const long long b = r / L;
  const int j = static_cast<int>(r - b * L);
  const bool is_ctx = j < nctx;
  const float* prow = pos + static_cast<size_t>(is_ctx ? ctx[j] : tgt[j - nctx]) * D;
  const float* srow = is_ctx ? e + (b * nctx + j) * D : mask;
  float* xrow = x + r * D;
  for (int c = threadIdx.x * 4; c < D; c += blockDim.x * 4) {
    const float4 u = *reinterpret_cast<const float4*>(srow + c), v = *reinterpret_cast<const float4*>(prow + c);
    *reinterpret_cast<float4*>(xrow + c) = make_float4(u.x + v.x, u.y + v.y, u.z + v.z, u.w + v.w);
  }
}

int launch_pred_assemble(const float* e, const float* mask, const float* pos, const int* ctx, const int* tgt, int B,
                         int nctx, int ntgt, int D, float* x, cudaStream_t st) {
  if (!e || !mask || !pos || !ctx || !tgt || !x) return JEPA_B200_ERR_ARG;
  if (B < 1 || nctx < 1 || ntgt < 1 || D < 4 || D % 4 != 0) return JEPA_B200_ERR_SHAPE;
  launch_pdl(pred_assemble_kernel, dim3(static_cast<unsigned>(B) * (nctx + ntgt)), dim3(128), 0, st, 1, e, mask, pos,
             ctx, tgt, nctx, ntgt, D, x);
  return cudaGetLastError() == cudaSuccess ? JEPA_B200_OK : JEPA_B200_ERR_CUDA;
}

// Mean pooling over rows first..ntok-1 of each clip, deterministic two-stage
// reduction: column sums over row chunks, then the chunk sums.
constexpr int kPoolSplits = 32;

__global__ void mean_pool_partial_kernel(const float* __restrict__ y, int ntok, int D, int first,
                                         float* __restrict__ partial) {
  pdl_wait();
  pdl_trigger();
  const int col = blockIdx.x * 256 + threadIdx.x;
  const int sp = blockIdx.y, b = blockIdx.z;
  if (col >= D) return;
  const int n_rows = ntok - first;
  const int per = (n_rows + kPoolSplits - 1) / kPoolSplits;
  const int r0 = first + sp * per, r1 = min(ntok, r0 + per);
  const float* base = y + static_cast<size_t>(b) * ntok * D + col;
  float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
  int r = r0;
  for (; r + 3 < r1; r += 4) {
    s0 += __ldg(base + static_cast<size_t>(r) * D);
    s1 += __ldg(base + static_cast<size_t>(r + 1) * D);
    s2 += __ldg(base + static_cast<size_t>(r + 2) * D);
    s3 += __ldg(base + static_cast<size_t>(r + 3) * D);
  }
  for (; r < r1; ++r) s0 += __ldg(base + static_cast<size_t>(r) * D);
  partial[(static_cast<size_t>(b) * kPoolSplits + sp) * D + col] = (s0 + s1) + (s2 + s3);
}

__global__ void mean_pool_final_kernel(const float* __restrict__ partial, int B, int D, float inv_count,
                                       float* __restrict__ out) {
  pdl_wait();
  pdl_trigger();
  const int i = blockIdx.x * 256 + threadIdx.x;
  if (i >= B * D) return;
  const int b = i / D, col = i % D;
  float s = 0.f;
  for (int sp = 0; sp < kPoolSplits; ++sp) s += partial[(static_cast<size_t>(b) * kPoolSplits + sp) * D + col];
  out[i] = s * inv_count;
}

int mean_pool_partial_floats(int B, int D) { return B * kPoolSplits * D; }

int launch_mean_pool(const float* y, int B, int ntok, int D, int first, float* partial, float* out,
                     cudaStream_t st) {
  if (!y || !partial || !out) return JEPA_B200_ERR_ARG;
  if (B < 1 || D < 1 || first < 0 || first >= ntok || B > 65535) return JEPA_B200_ERR_SHAPE;
  launch_pdl(mean_pool_partial_kernel, dim3((D + 255) / 256, kPoolSplits, B), dim3(256), 0, st, 1, y, ntok, D, first,
             partial);
  launch_pdl(mean_pool_final_kernel, dim3((B * D + 255) / 256), dim3(256), 0, st, 1, static_cast<const float*>(partial),
             B, D, 1.0f / (ntok - first), out);
  return cudaGetLastError() == cudaSuccess ? JEPA_B200_OK : JEPA_B200_ERR_CUDA;
}

// Repack [N, K/32] q8_0 (34-byte) or q4_0 (18-byte) blocks into
// qs [N, K] int8 or [N, K/2] nibble bytes (block order kept) + scales [N, K/32].
__global__ void repack_kernel(int bmode, const uint8_t* __restrict__ blocks, long long nblocks, uint8_t* qs,
                              uint16_t* scales) {
  pdl_wait();
  pdl_trigger();
  const long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= nblocks) return;
  const int bsz = bmode == B_Q8 ? 34 : 18;
  const int qbytes = bmode == B_Q8 ? 32 : 16;
  const uint8_t* src = blocks + i * bsz;
  scales[i] = static_cast<uint16_t>(src[0] | (src[1] << 8));
  uint8_t* dst = qs + i * qbytes;
  for (int j = 0; j < qbytes; ++j) dst[j] = src[2 + j];
}

int launch_repack(int bmode, const uint8_t* blocks, int N, int K, void* qs, __half* scales, cudaStream_t st) {
  if (!blocks || !qs || !scales) return JEPA_B200_ERR_ARG;
  if ((bmode != B_Q8 && bmode != B_Q4) || N < 1 || K < 32 || K % 32 != 0) return JEPA_B200_ERR_SHAPE;
  const long long nb = static_cast<long long>(N) * (K / 32);
  repack_kernel<<<static_cast<unsigned>((nb + 255) / 256), 256, 0, st>>>(
      bmode, blocks, nb, static_cast<uint8_t*>(qs), reinterpret_cast<uint16_t*>(scales));
  return cudaGetLastError() == cudaSuccess ? JEPA_B200_OK : JEPA_B200_ERR_CUDA;
}

// f16 copy of a repacked matrix: element (n, k) = q * d (q8_0) or (q - 8) * d
// (q4_0), d the scale of its 32-element block; the product is exact in f32
// (an 8-bit integer times an 11-bit significand) and rounded once to f16.
// One thread writes 8 consecutive elements of one block.
template <bool BF>
__global__ void dequant_f16_kernel(int bmode, const uint8_t* __restrict__ qs, const uint16_t* __restrict__ scales,
                                   long long n_units, int K, __half* __restrict__ out) {
  pdl_wait();
  pdl_trigger();
  const long long u = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (u >= n_units) return;
  const long long e0 = u * 8;  // first element, row-major [N, K]
  const long long n = e0 / K;
  const int k = static_cast<int>(e0 - n * K);
  const float d = __half2float(__ushort_as_half(scales[n * (K / 32) + k / 32]));
  float v[8];
  if (bmode == B_Q8) {
    const int8_t* q = reinterpret_cast<const int8_t*>(qs) + e0;
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = static_cast<float>(q[i]) * d;
  } else {
    const int j0 = k & 31;  // byte j of a block holds elements j (low nibble) and j + 16 (high)
    const uint8_t* q = qs + n * (K / 2) + (k / 32) * 16 + (j0 & 15);
    const int sh = j0 >= 16 ? 4 : 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = static_cast<float>(static_cast<int>((q[i] >> sh) & 0xF) - 8) * d;
  }
  uint4 w;
  w.x = pack2<BF>(v[0], v[1]);
  w.y = pack2<BF>(v[2], v[3]);
  w.z = pack2<BF>(v[4], v[5]);
  w.w = pack2<BF>(v[6], v[7]);
  *reinterpret_cast<uint4*>(out + e0) = w;
}

int launch_dequant_f16(int bmode, const void* qs, const __half* scales, int N, int K, __half* out, cudaStream_t st,
                       bool bf16) {
  if (!qs || !scales || !out) return JEPA_B200_ERR_ARG;
  if ((bmode != B_Q8 && bmode != B_Q4) || N < 1 || K < 32 || K % 32 != 0) return JEPA_B200_ERR_SHAPE;
  const long long units = static_cast<long long>(N) * K / 8;
  launch_pdl(bf16 ? dequant_f16_kernel<true> : dequant_f16_kernel<false>,
             dim3(static_cast<unsigned>((units + 255) / 256)), dim3(256), 0, st, 1, bmode,
             static_cast<const uint8_t*>(qs), reinterpret_cast<const uint16_t*>(scales), units, K, out);
  return cudaGetLastError() == cudaSuccess ? JEPA_B200_OK : JEPA_B200_ERR_CUDA;
}

}  // namespace jb
