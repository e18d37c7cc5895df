// Flash attention on tcgen05 for the JEPA encoders, head dim 64.
//
// O = softmax(Q K^T / sqrt(64) + mask) V per (clip, head).  The mask is
// either none (V-JEPA 2, LeWM: bidirectional) or LeVJEPA's block-causal mask
// ("LeVJEPA ViT-L/16 (VideoMix) -- GGUF for jepa.cpp", intro: bidirectional
// inside a frame, causal across frames, the CLS token a read-only sink).  For
// every query row the allowed keys form one interval [lo, hi]:
//   CLS row:            [0, N-1]
//   patch of slot s:    [c, c + (s+1) * P_f - 1]   (c = 1 with a CLS row)
// so a query tile only visits KV tiles up to its largest hi; tiles past it
// are never loaded (the skipped, fully masked tiles).
//
// One CTA per (128-query tile, clip*head); two CTAs per SM so one CTA's
// softmax overlaps the other's tensor-core work.
//   warp 0     TMA: Q tile once, K tiles (2 stages) and V^T tiles;
//   warp 1     MMA: S = Q K^T into TMEM (M=128, N=128), then O += P V into
//              TMEM (M=128, N=64) with P from shared memory;
//   warps 2-5  softmax, one thread per query row: row max from TMEM, O
//              rescaled in TMEM when the max grows, P = exp2(.) written as
//              f16 into the swizzled A tile of the PV product, row sum in f32;
//              at the end O / l is written token-major for the out-projection.
#include <string.h>

#include <algorithm>

#include "internal.h"

namespace jb {

namespace {
constexpr int kQBytes = 128 * 64 * 2;   // Q tile [128 x 64]
constexpr int kKBytes = 128 * 64 * 2;   // K tile [128 keys x 64]
constexpr int kVBytes = 64 * 128 * 2;   // V^T tile [64 dims x 128 keys] as two [64 x 64] halves
constexpr int kPBytes = 128 * 128 * 2;  // P tile [128 x 128 keys] as two [128 x 64] halves
constexpr int kAttnSmem = kQBytes + 2 * kKBytes + kVBytes + kPBytes + 1024;
}  // namespace

__device__ __forceinline__ void key_range(const AttnParams& p, int i, int& lo, int& hi) {
  lo = 0;
  hi = p.N - 1;
  if (p.mask == JEPA_B200_MASK_BLOCK_CAUSAL && i < p.N) {
    if (p.has_cls) {
      if (i > 0) {
        const int s = (i - 1) / p.ppf;
        lo = 1;
        hi = (s + 1) * p.ppf;
      }
    } else {
      const int s = i / p.ppf;
      hi = (s + 1) * p.ppf - 1;
    }
    if (hi > p.N - 1) hi = p.N - 1;
  }
}

__global__ void __launch_bounds__(192, 2)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const AttnParams p) {
  extern __shared__ uint8_t dsmem[];
  __shared__ uint64_t q_full, k_full[2], k_empty[2], v_full, v_empty, s_full, p_full, pv_done, drain_bar;
  __shared__ uint32_t tmem_sh;
  __shared__ int abort_sh;

  const uint32_t raw = smem_u32(dsmem);
  uint8_t* sm = dsmem + ((1024u - (raw & 1023u)) & 1023u);
  uint8_t* sQ = sm;
  uint8_t* sK0 = sm + kQBytes;
  uint8_t* sV = sK0 + 2 * kKBytes;
  uint8_t* sP = sV + kVBytes;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qt = p.n_q_tiles - 1 - static_cast<int>(blockIdx.x);  // late (heavier) tiles first
  const int bh = blockIdx.y;
  const int q0 = qt * 128;

  // KV tiles this query tile needs: up to the largest hi over its rows.
  int lo_a, hi_a, lo_b, hi_b;
  key_range(p, q0, lo_a, hi_a);
  key_range(p, min(q0 + 127, p.N - 1), lo_b, hi_b);
  const int kv_end = max(hi_a, hi_b) + 1;
  const int n_kv = (kv_end + 127) / 128;

  if (threadIdx.x == 0) {
    mbar_init(&q_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&k_empty[i], 1);
    }
    mbar_init(&v_full, 1);
    mbar_init(&v_empty, 1);
    mbar_init(&s_full, 1);
    mbar_init(&p_full, 128);
    mbar_init(&pv_done, 1);
    mbar_init(&drain_bar, 1);
    abort_sh = 0;
    mbar_fence_init();
  }
  if (warp == 1) {
    tmem_alloc(&tmem_sh, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tS = tmem_sh;         // S: columns 0..127
  const uint32_t tO = tmem_sh + 128;   // O: columns 128..191

  WaitCtl w;
  w.abort = reinterpret_cast<volatile int*>(&abort_sh);
  w.err = p.err;
  w.timeout_ns = p.timeout_ns;
  w.where = (KID_ATTN << 8) | static_cast<unsigned>(warp);

  if (warp == 0) {
    if (lane == 0) {
      bool ok = true;
      uint32_t karmed = 0, kpar = 0, varmed = 0, vpar = 0;
      mbar_expect_tx(&q_full, kQBytes);
      tma_load_3d(sQ, &tmQ, &q_full, 0, q0, bh);
      for (int j = 0; j < n_kv; ++j) {
        const int ks = j & 1;
        const uint32_t kph = (j >> 1) & 1;
        if (!mbar_wait(&k_empty[ks], kph ^ 1, w)) {
          ok = false;
          break;
        }
        mbar_expect_tx(&k_full[ks], kKBytes);
        tma_load_3d(sK0 + ks * kKBytes, &tmK, &k_full[ks], 0, j * 128, bh);
        karmed |= 1u << ks;
        kpar = (kpar & ~(1u << ks)) | (kph << ks);
        if (!mbar_wait(&v_empty, (j & 1) ^ 1, w)) {
          ok = false;
          break;
        }
        mbar_expect_tx(&v_full, kVBytes);
        tma_load_3d(sV, &tmV, &v_full, j * 128, 0, bh);
        tma_load_3d(sV + kVBytes / 2, &tmV, &v_full, j * 128 + 64, 0, bh);
        varmed = 1;
        vpar = j & 1;
      }
      if (!ok) {
        mbar_wait_drain(&q_full, 0);
        for (int s = 0; s < 2; ++s)
          if ((karmed >> s) & 1u) mbar_wait_drain(&k_full[s], (kpar >> s) & 1u);
        if (varmed) mbar_wait_drain(&v_full, vpar);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_f16_f32(128, 128);
      constexpr uint32_t idesc_o = idesc_f16_f32(128, 64);
      const uint64_t qd = sdesc_kmajor_sw128(smem_u32(sQ));
      const uint64_t pd0 = sdesc_kmajor_sw128(smem_u32(sP));
      const uint64_t pd1 = sdesc_kmajor_sw128(smem_u32(sP + kPBytes / 2));
      const uint64_t vd0 = sdesc_kmajor_sw128(smem_u32(sV));
      const uint64_t vd1 = sdesc_kmajor_sw128(smem_u32(sV + kVBytes / 2));
      bool ok = mbar_wait(&q_full, 0, w);
      // O += P_j V_j (j = tile index), after softmax published P_j
      auto issue_pv = [&](int j) -> bool {
        if (!mbar_wait(&p_full, j & 1, w)) return false;
        if (!mbar_wait(&v_full, j & 1, w)) return false;
        tc_fence_after();
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const uint64_t ad = (k < 4 ? pd0 : pd1) + static_cast<uint64_t>(2 * (k & 3));
          const uint64_t bd = (k < 4 ? vd0 : vd1) + static_cast<uint64_t>(2 * (k & 3));
          tc_mma_f16_ss(tO, ad, bd, idesc_o, (j > 0 || k > 0) ? 1u : 0u);
        }
        tc_commit(&v_empty);
        tc_commit(&pv_done);
        return true;
      };
      for (int j = 0; ok && j < n_kv; ++j) {
        const int ks = j & 1;
        if (!mbar_wait(&k_full[ks], (j >> 1) & 1, w)) {
          ok = false;
          break;
        }
        // S is free once softmax published P_{j-1} (it has read S_{j-1})
        if (j > 0 && !mbar_wait(&p_full, (j - 1) & 1, w)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint64_t kd = sdesc_kmajor_sw128(smem_u32(sK0 + ks * kKBytes));
#pragma unroll
        for (int k = 0; k < 4; ++k)
          tc_mma_f16_ss(tS, qd + static_cast<uint64_t>(2 * k), kd + static_cast<uint64_t>(2 * k), idesc_s,
                        k > 0 ? 1u : 0u);
        tc_commit(&k_empty[ks]);
        tc_commit(&s_full);
        if (j > 0 && !issue_pv(j - 1)) {
          ok = false;
          break;
        }
      }
      if (ok) issue_pv(n_kv - 1);
      tc_commit(&drain_bar);
      mbar_wait_drain(&drain_bar, 0);
    }
  } else {
    // softmax: one thread per query row
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    const int i = q0 + r;
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    int lo, hi;
    key_range(p, i, lo, hi);
    if (i >= p.N) {
      lo = 0;
      hi = p.N - 1;
    }
    const float sc = p.scale_log2;
    float m_run = -INFINITY, l_run = 0.0f;
    const uint32_t pbase = smem_u32(sP);
    bool ok = true;
    for (int j = 0; j < n_kv; ++j) {
      bool okw = mbar_wait(&s_full, j & 1, w);
      okw = __all_sync(0xffffffffu, okw);
      if (!okw) {
        ok = false;
        break;
      }
      tc_fence_after();
      const int kbase = j * 128;
      // pass 1: masked row max of the scaled scores (log2 domain)
      float mx = -INFINITY;
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        uint32_t s[32];
        tmem_ld32(tS + lane_off + static_cast<uint32_t>(c * 32), s);
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const int key = kbase + c * 32 + e;
          const float v = __uint_as_float(s[e]) * sc;
          if (key >= lo && key <= hi) mx = fmaxf(mx, v);
        }
      }
      const float m_new = fmaxf(m_run, mx);
      if (j > 0) {  // P buffer free and O stable once PV_{j-1} is done
        okw = mbar_wait(&pv_done, (j - 1) & 1, w);
        okw = __all_sync(0xffffffffu, okw);
        if (!okw) {
          ok = false;
          break;
        }
        tc_fence_after();
        // tcgen05.ld / st are warp-collective: the whole warp rescales its
        // rows when any of them saw a larger max (the others scale by 1).
        const bool grow = m_new > m_run && m_run != -INFINITY;
        if (__any_sync(0xffffffffu, grow)) {
          const float alpha = grow ? ex2_approx(m_run - m_new) : 1.0f;
          l_run *= alpha;
#pragma unroll 1
          for (int c = 0; c < 2; ++c) {
            uint32_t o[32];
            tmem_ld32(tO + lane_off + static_cast<uint32_t>(c * 32), o);
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
            tmem_st32(tO + lane_off + static_cast<uint32_t>(c * 32), o);
          }
        }
      }
      // a row may still see no allowed key (m = -inf): then every p is 0
      m_run = m_new;
      const float m_use = m_run == -INFINITY ? 0.0f : m_run;
      // pass 2: P = exp2(s - m), row sum, f16 into the swizzled P tile
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        uint32_t s[32];
        tmem_ld32(tS + lane_off + static_cast<uint32_t>(c * 32), s);
        uint32_t h[16];
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          const int key = kbase + c * 32 + e;
          float pa = 0.0f, pb = 0.0f;
          if (key >= lo && key <= hi) pa = ex2_approx(__uint_as_float(s[e]) * sc - m_use);
          if (key + 1 >= lo && key + 1 <= hi) pb = ex2_approx(__uint_as_float(s[e + 1]) * sc - m_use);
          l_run += pa + pb;
          h[e >> 1] = pack_half2(pa, pb);
        }
        const uint32_t half_base = pbase + static_cast<uint32_t>((c >> 1) * (kPBytes / 2));
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int kk = (c & 1) * 32 + u * 8;
          st_shared_v4(half_base + sw128_offset(r, kk), h[4 * u], h[4 * u + 1], h[4 * u + 2], h[4 * u + 3]);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&p_full);
    }
    if (ok) {
      bool okw = mbar_wait(&pv_done, (n_kv - 1) & 1, w);
      okw = __all_sync(0xffffffffu, okw);
      if (okw) {
        tc_fence_after();
        const float inv_l = l_run > 0.0f ? 1.0f / l_run : 0.0f;
        const int b = bh / p.heads, hd = bh % p.heads;
#pragma unroll 1
        for (int c = 0; c < 2; ++c) {
          uint32_t o[32];
          tmem_ld32(tO + lane_off + static_cast<uint32_t>(c * 32), o);
          if (i < p.N) {
            uint4* dst = reinterpret_cast<uint4*>(p.out + (static_cast<size_t>(b) * p.N + i) * p.ldo + hd * 64 + c * 32);
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const float* f = reinterpret_cast<const float*>(o) + 8 * u;
              dst[u] = make_uint4(pack_half2(f[0] * inv_l, f[1] * inv_l), pack_half2(f[2] * inv_l, f[3] * inv_l),
                                  pack_half2(f[4] * inv_l, f[5] * inv_l), pack_half2(f[6] * inv_l, f[7] * inv_l));
            }
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_sh, 256);
  }
}

int attn_prepare(AttnOp* op, const __half* q, const __half* k, const __half* vt, int B, int heads, int ntok,
                 int npad, int mask, int has_cls, int ppf, __half* out) {
  if (!op || !q || !k || !vt || !out) return JEPA_B200_ERR_ARG;
  if (B < 1 || heads < 1 || ntok < 1 || npad < ntok || npad % 128 != 0) return JEPA_B200_ERR_SHAPE;
  if (mask != JEPA_B200_MASK_BIDIR && mask != JEPA_B200_MASK_BLOCK_CAUSAL) return JEPA_B200_ERR_ARG;
  if (mask == JEPA_B200_MASK_BLOCK_CAUSAL && (ppf < 1 || (ntok - (has_cls ? 1 : 0)) % ppf != 0))
    return JEPA_B200_ERR_SHAPE;
  if (static_cast<long long>(B) * heads > 65535) return JEPA_B200_ERR_SHAPE;
  memset(op, 0, sizeof(*op));
  const uint64_t BH = static_cast<uint64_t>(B) * heads;
  {
    const uint64_t dims[3] = {64, static_cast<uint64_t>(ntok), BH};
    const uint64_t str[2] = {128, static_cast<uint64_t>(ntok) * 128};
    const uint32_t box[3] = {64, 128, 1};
    if (!make_tmap_f16(&op->tmQ, q, 3, dims, str, box)) return JEPA_B200_ERR_CUDA;
    if (!make_tmap_f16(&op->tmK, k, 3, dims, str, box)) return JEPA_B200_ERR_CUDA;
  }
  {
    const uint64_t dims[3] = {static_cast<uint64_t>(npad), 64, BH};
    const uint64_t str[2] = {static_cast<uint64_t>(npad) * 2, static_cast<uint64_t>(npad) * 128};
    const uint32_t box[3] = {64, 64, 1};
    if (!make_tmap_f16(&op->tmV, vt, 3, dims, str, box)) return JEPA_B200_ERR_CUDA;
  }
  AttnParams& p = op->p;
  p.N = ntok;
  p.heads = heads;
  p.n_q_tiles = (ntok + 127) / 128;
  p.mask = mask;
  p.has_cls = has_cls ? 1 : 0;
  p.ppf = ppf < 1 ? 1 : ppf;
  p.scale_log2 = 1.4426950408889634f / 8.0f;
  p.out = out;
  p.ldo = heads * 64;
  op->B = B;
  op->smem = kAttnSmem;
  return JEPA_B200_OK;
}

int attn_launch(const AttnOp& op, cudaStream_t st, DevErr* err, unsigned long long timeout_ns) {
  static unsigned long long attr_done = 0;
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !((attr_done >> dev) & 1ull)) {
    if (cudaFuncSetAttribute(attn_fwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kAttnSmem) !=
        cudaSuccess)
      return JEPA_B200_ERR_CUDA;
    attr_done |= 1ull << dev;
  }
  AttnParams p = op.p;
  p.err = err;
  p.timeout_ns = timeout_ns;
  dim3 grid(p.n_q_tiles, op.B * p.heads);
  attn_fwd_kernel<<<grid, 192, kAttnSmem, st>>>(op.tmQ, op.tmK, op.tmV, p);
  return cudaGetLastError() == cudaSuccess ? JEPA_B200_OK : JEPA_B200_ERR_CUDA;
}

}  // namespace jb
