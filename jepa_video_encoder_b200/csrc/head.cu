// Kernels of the attentive-pool classifier head ("jepa.cpp -- measured
// benchmarks", section "Attentive-pool head": 3 self-attention blocks over
// the tokens, one cross-attention query, MLP, linear; the 174-class SSv2 head
// of "V-JEPA 2 ViT-L/16 SSv2 classifier -- GGUF for jepa.cpp").  The
// self-attention blocks reuse the encoder's kernels; what is left has one
// row per clip (the single query), so it is matrix-vector work bound by the
// weight stream:
//   gemv:      y = epi(x W^T + b) for a few rows, f16 / q8_0 / q4_0 weights
//              unpacked in registers;
//   xattn_1q:  one learned query against all N keys of a clip, per head.
#include <algorithm>

#include "internal.h"

namespace jb {

__device__ __forceinline__ float warp_sum_h(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max_h(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

constexpr int kGemvRows = 8;

// 8 consecutive weights of row n starting at k (k a multiple of 8); 16-bit
// weights are f16, or bf16 (BF).
template <int BMODE, bool BF>
__device__ __forceinline__ void load_w8(const void* __restrict__ w, const __half* __restrict__ scales, int K, int n,
                                        int k, float (&o)[8]) {
  if (BMODE == B_F16) {
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(static_cast<const __half*>(w) + static_cast<size_t>(n) * K + k));
    const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      o[2 * e] = widen1<BF>(static_cast<unsigned short>(u[e] & 0xFFFFu));
      o[2 * e + 1] = widen1<BF>(static_cast<unsigned short>(u[e] >> 16));
    }
  } else {
    const float d = __half2float(scales[static_cast<size_t>(n) * (K >> 5) + (k >> 5)]);
    if (BMODE == B_Q8) {
      const uint2 q = __ldg(reinterpret_cast<const uint2*>(static_cast<const int8_t*>(w) + static_cast<size_t>(n) * K + k));
      const uint32_t qq[2] = {q.x, q.y};
#pragma unroll
      for (int e = 0; e < 8; ++e)
        o[e] = static_cast<float>(static_cast<int8_t>((qq[e >> 2] >> ((e & 3) * 8)) & 0xFF)) * d;
    } else {
      const int j0 = k & 31;
      const uint2 q = __ldg(reinterpret_cast<const uint2*>(static_cast<const uint8_t*>(w) +
                                                           static_cast<size_t>(n) * (K >> 1) + (k >> 5) * 16 +
                                                           (j0 & 15)));
      const int nsh = j0 >= 16 ? 4 : 0;
      const uint32_t qq[2] = {q.x, q.y};
#pragma unroll
      for (int e = 0; e < 8; ++e)
        o[e] = static_cast<float>(static_cast<int>((qq[e >> 2] >> ((e & 3) * 8 + nsh)) & 0xF) - 8) * d;
    }
  }
}

template <int BMODE, bool BF>
__global__ void __launch_bounds__(256) gemv_kernel(const float* __restrict__ x, int M, int K,
                                                  const void* __restrict__ w, const __half* __restrict__ scales,
                                                  int N, const float* __restrict__ bias, int epi, const float* resid,
                                                  long long resid_stride, float* y) {
  extern __shared__ float xs[];
  pdl_wait();
  pdl_trigger();
  for (int i = threadIdx.x; i < M * K; i += 256) xs[i] = x[i];
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n = blockIdx.x * 8 + warp;
  if (n >= N) return;
  float acc[kGemvRows];
#pragma unroll
  for (int m = 0; m < kGemvRows; ++m) acc[m] = 0.0f;
  for (int k = lane * 8; k < K; k += 256) {
    float wv[8];
    load_w8<BMODE, BF>(w, scales, K, n, k, wv);
#pragma unroll
    for (int m = 0; m < kGemvRows; ++m) {
      if (m < M) {
        const float* xr = xs + m * K + k;
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[m] = fmaf(wv[e], xr[e], acc[m]);
      }
    }
  }
#pragma unroll
  for (int m = 0; m < kGemvRows; ++m) {
    if (m < M) {
      float v = warp_sum_h(acc[m]);
      if (lane == 0) {
        if (bias) v += bias[n];
        if (epi == 1) v = gelu1(v);
        if (epi == 2) v += resid[static_cast<size_t>(m) * resid_stride + n];
        y[static_cast<size_t>(m) * N + n] = v;
      }
    }
  }
}

int launch_gemv(const float* x, int M, int K, const DevMatrix& W, const float* bias, int epi, const float* resid,
                long long resid_stride, float* y, cudaStream_t st) {
  if (!x || !y || !W.data) return JEPA_B200_ERR_ARG;
  if (M < 1 || K < 8 || K % 8 != 0 || W.K != K || W.N < 1) return JEPA_B200_ERR_SHAPE;
  if (W.bmode != B_F16 && (K % 32 != 0 || !W.scales)) return JEPA_B200_ERR_SHAPE;
  if (epi == 2 && !resid) return JEPA_B200_ERR_ARG;
  const int N = W.N;
  int rows_per = kGemvRows;
  while (rows_per > 1 && static_cast<size_t>(rows_per) * K * 4 > 200 * 1024) rows_per >>= 1;
  if (static_cast<size_t>(K) * 4 > 200 * 1024) return JEPA_B200_ERR_SHAPE;
  const int smem_max = rows_per * K * 4;
  static std::atomic<unsigned long long> attr_done[4] = {};
  const int bm = W.bmode == B_Q8 ? 1 : (W.bmode == B_Q4 ? 2 : (W.bf16 ? 3 : 0));
  const bool attr_ok = bm == 1   ? smem_attr_once(attr_done[1], gemv_kernel<B_Q8, false>, 200 * 1024)
                       : bm == 2 ? smem_attr_once(attr_done[2], gemv_kernel<B_Q4, false>, 200 * 1024)
                       : bm == 3 ? smem_attr_once(attr_done[3], gemv_kernel<B_F16, true>, 200 * 1024)
                                 : smem_attr_once(attr_done[0], gemv_kernel<B_F16, false>, 200 * 1024);
  if (!attr_ok) return JEPA_B200_ERR_CUDA;
  (void)smem_max;
  for (int m0 = 0; m0 < M; m0 += rows_per) {
    const int mc = std::min(rows_per, M - m0);
    const dim3 grid((N + 7) / 8);
    const size_t smem = static_cast<size_t>(mc) * K * 4;
    const float* xr = x + static_cast<size_t>(m0) * K;
    const float* rr = resid ? resid + static_cast<size_t>(m0) * resid_stride : nullptr;
    float* yr = y + static_cast<size_t>(m0) * N;
    auto kern = bm == 1 ? gemv_kernel<B_Q8, false>
              : bm == 2 ? gemv_kernel<B_Q4, false>
              : bm == 3 ? gemv_kernel<B_F16, true>
                        : gemv_kernel<B_F16, false>;
    launch_pdl(kern, grid, dim3(256), smem, st, 1, xr, mc, K, static_cast<const void*>(W.data),
               static_cast<const __half*>(W.scales), N, bias, epi, rr, resid_stride, yr);
  }
  return cudaGetLastError() == cudaSuccess ? JEPA_B200_OK : JEPA_B200_ERR_CUDA;
}

// One query per (clip, head) over all ntok keys: softmax(q k^T / 8) v.
template <bool BF>
__global__ void __launch_bounds__(256) xattn_1q_kernel(const float* __restrict__ q, const __half* __restrict__ k,
                                                       const __half* __restrict__ vt, int heads, int ntok, int npad,
                                                       float* __restrict__ out) {
  extern __shared__ float sc[];
  __shared__ float qh[64];
  pdl_wait();
  pdl_trigger();
  __shared__ float red[8];
  const int bh = blockIdx.x, b = bh / heads, hd = bh % heads;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x < 64) qh[threadIdx.x] = q[hd * 64 + threadIdx.x];
  __syncthreads();
  const __half* kb = k + static_cast<size_t>(bh) * ntok * 64;
  float mx = -INFINITY;
  for (int j = threadIdx.x; j < ntok; j += 256) {
    const uint4* kr = reinterpret_cast<const uint4*>(kb + static_cast<size_t>(j) * 64);
    float s = 0.0f;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const uint4 v = __ldg(kr + u);
      const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        s = fmaf(qh[u * 8 + 2 * e], widen1<BF>(static_cast<unsigned short>(w4[e] & 0xFFFFu)), s);
        s = fmaf(qh[u * 8 + 2 * e + 1], widen1<BF>(static_cast<unsigned short>(w4[e] >> 16)), s);
      }
    }
    s *= 0.125f;
    sc[j] = s;
    mx = fmaxf(mx, s);
  }
  mx = warp_max_h(mx);
  if (lane == 0) red[warp] = mx;
  __syncthreads();
  float M = red[0];
  for (int i = 1; i < 8; ++i) M = fmaxf(M, red[i]);
  __syncthreads();
  float l = 0.0f;
  for (int j = threadIdx.x; j < ntok; j += 256) {
    const float p = __expf(sc[j] - M);
    sc[j] = p;
    l += p;
  }
  l = warp_sum_h(l);
  if (lane == 0) red[warp] = l;
  __syncthreads();
  float L = 0.0f;
  for (int i = 0; i < 8; ++i) L += red[i];
  const float invL = 1.0f / L;
  for (int d = warp; d < 64; d += 8) {
    const __half* vr = vt + (static_cast<size_t>(bh) * 64 + d) * npad;
    float acc = 0.0f;
    for (int j = lane; j < ntok; j += 32) acc = fmaf(sc[j], widen1<BF>(__half_as_ushort(vr[j])), acc);
    acc = warp_sum_h(acc);
    if (lane == 0) out[static_cast<size_t>(b) * heads * 64 + hd * 64 + d] = acc * invL;
  }
}

int launch_xattn_1q(const float* q, const __half* k, const __half* vt, int B, int heads, int ntok, int npad,
                    float* out, cudaStream_t st, bool bf16) {
  if (!q || !k || !vt || !out) return JEPA_B200_ERR_ARG;
  if (B < 1 || heads < 1 || ntok < 1 || ntok > 16384 || npad < ntok) return JEPA_B200_ERR_SHAPE;
  const size_t smem = static_cast<size_t>(ntok) * 4;
  static std::atomic<unsigned long long> attr_done[2] = {};
  auto kern = bf16 ? xattn_1q_kernel<true> : xattn_1q_kernel<false>;
  if (!smem_attr_once(attr_done[bf16 ? 1 : 0], kern, 16384 * 4)) return JEPA_B200_ERR_CUDA;
  launch_pdl(kern, dim3(B * heads), dim3(256), smem, st, 1, q, k, vt, heads, ntok, npad, out);
  return cudaGetLastError() == cudaSuccess ? JEPA_B200_OK : JEPA_B200_ERR_CUDA;
}

}  // namespace jb
