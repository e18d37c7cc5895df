// Flash attention on tcgen05 for the JEPA encoders, head dim 64.
//
// O = softmax(Q K^T / sqrt(64) + mask) V per (clip, head).  The mask is
// either none (V-JEPA 2, LeWM: bidirectional) or LeVJEPA's block-causal mask
// ("LeVJEPA ViT-L/16 (VideoMix) -- GGUF for jepa.cpp", intro: bidirectional
// inside a frame, causal across frames, the CLS token a read-only sink).  For
// every query row the allowed keys form one interval [lo, hi]:
//   CLS row:            [0, N-1]
//   patch of slot s:    [c, c + (s+1) * P_f - 1]   (c = 1 with a CLS row)
// so a query tile only visits KV tiles up to its largest hi (the fully masked
// tiles past it are never loaded), and only tiles that cut an interval need
// the per-element mask.  The CLS row, the one row that reads every key, is
// computed apart so that query tile 0 stays as short as the first frame's:
// with one query tile per CTA and N % 128 != 0, its query is copied into row
// N (the first padding row) of the last query tile, which already visits
// every KV tile; otherwise a "CLS tile" (the query tile at row 0 against
// every KV tile, only row 0 kept) runs as the second tile of the last pair
// (two tiles per CTA, odd tile count) or in a CTA of its own.
//
// Bidirectional: one CTA per (pair of 128-query tiles, clip*head), one CTA
// per SM.  Block-causal: one CTA per (128-query tile, clip*head), two CTAs
// per SM (half the TMEM and shared memory each), so that the start and the
// drain of one CTA's short tile overlap the other CTA's work.
//   warp 0      TMA: the Q tile(s) once, then K and V^T tiles through a
//               ring (4 stages shared by the two query tiles, or 2);
//   warps 1,18  MMA, one issuer per query tile g (warp 18 with two tiles): for each KV tile j,
//               S_g = Q_g K_j^T into TMEM (M=128, N=128, both operands in
//               shared memory) and O_g += P_g V_{j-1} into TMEM (M=128, N=64,
//               P read from TMEM);
//   warps 2-9   softmax of query tile 0, warps 10-17 of query tile 1:
//               scores read once from TMEM into registers (S is released at
//               once for the next KV tile), O rescaled in TMEM only when the
//               row max grew by more than 2^8 (lazy rescaling: P stays <= 256,
//               exact after the final division by the row sum), P =
//               exp2(s*c - m) packed as f16 pairs into TMEM for the PV
//               product.  Two row layouts (template ROWS_IN_WARP):
//                 bidirectional: two threads per row in two warps of a lane
//                 quadrant (32x32b TMEM shape), each with 64 keys, row max
//                 and sum combined through shared memory;
//                 block-causal: four threads per row in one warp (16x256b /
//                 16x128b TMEM shapes), each with 32 keys of two rows, row
//                 max and sum combined with shuffles -- no cross-warp barrier
//                 per KV tile, which dominates the short block-causal tiles.
#include <string.h>

#include <algorithm>
#include <cmath>

#include "internal.h"

namespace jb {

namespace {
constexpr int kTile = 128 * 64 * 2;  // one [128 x 64] f16 tile, 16 KB
constexpr float kRescaleLog2 = 8.0f;  // rescale O when the row max grew by more than 2^8
// Query tiles per CTA: 2 (one CTA per SM, K / V shared by the two tiles) or 1
// (two CTAs per SM, so one CTA's start and drain overlap the other's work).
template <int TILES>
struct AttnCfg {
  static constexpr int kStages = TILES == 2 ? 4 : 2;
  static constexpr int kOffQ = 0;                        // Q tiles
  static constexpr int kOffK = kOffQ + TILES * kTile;    // K ring
  static constexpr int kOffV = kOffK + kStages * kTile;  // V^T ring, each [64 dims x 128 keys] as two [64 x 64]
  static constexpr int kSmem = kOffV + kStages * kTile + 1024;
  // TMEM columns: S_g (f32, 128 keys), O_g (f32, 64 dims), P_g (f16 pairs, 128 keys)
  static constexpr uint32_t kColS = 0, kColO = 128 * TILES, kColP = 192 * TILES;
  static constexpr uint32_t kTmemCols = 256 * TILES;
  // producer, one MMA issuer per tile, 8 softmax warps per tile
  static constexpr int kThreads = (TILES == 2 ? 19 : 10) * 32;
};
}  // namespace

__device__ __forceinline__ void key_range(const AttnParams& p, int i, int& lo, int& hi) {
  lo = 0;
  hi = p.N - 1;
  if (p.mask == JEPA_B200_MASK_BLOCK_CAUSAL && i < p.N) {
    if (p.has_cls) {
      // row 0 (CLS) reads every key; its own CTA computes it, and in the
      // pair CTAs it takes slot 0's range so that its tile stays short
      const int s = i > 0 ? (i - 1) / p.ppf : 0;
      lo = 1;
      hi = (s + 1) * p.ppf;
    } else {
      const int s = i / p.ppf;
      hi = (s + 1) * p.ppf - 1;
    }
    if (hi > p.N - 1) hi = p.N - 1;
  }
}

// Number of KV tiles query tile starting at q0 must visit (0: no valid row).
__device__ __forceinline__ int kv_tiles(const AttnParams& p, int q0) {
  if (q0 >= p.N) return 0;
  int lo_a, hi_a, lo_b, hi_b;
  key_range(p, q0, lo_a, hi_a);
  key_range(p, min(q0 + 127, p.N - 1), lo_b, hi_b);
  return (max(hi_a, hi_b) + 1 + 127) / 128;
}

// Allowed keys of tile row i in this CTA: rows past N (padding) and, in
// the CLS CTA, row 0 take every key.
__device__ __forceinline__ void row_keys(const AttnParams& p, bool cls_tile, int i, int& lo, int& hi) {
  key_range(p, i, lo, hi);
  if (i >= p.N || cls_tile) {
    lo = 0;
    hi = p.N - 1;
  }
}

template <bool ROWS_IN_WARP, int TILES, bool BF>
__global__ void __launch_bounds__(AttnCfg<TILES>::kThreads, TILES == 2 ? 1 : 2)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const AttnParams p) {
  using C = AttnCfg<TILES>;
  constexpr int kStages = C::kStages;
  extern __shared__ uint8_t dsmem[];
  __shared__ uint64_t q_full, k_full[kStages], k_empty[kStages], v_full[kStages], v_empty[kStages];
  // per query tile g: S ready / S taken / P written / PV done
  __shared__ uint64_t s_full[2], s_free[2], p_full[2], pv_done[2], drain_bar[2];
  __shared__ uint64_t stagger_bar;  // one phase: query tile 0 has computed its first P (cross-warp layout)
  // cross-warp row layout only: both halves of every row posted their partial
  __shared__ uint64_t x_bar[2];
  __shared__ float xmax[2][2][2][128];  // [tile parity][g][column half][row]: partial row maxima
  __shared__ float xsum[2][2][128];     // [g][column half][row]: partial row sums
  __shared__ uint32_t tmem_sh;
  __shared__ int abort_sh;

  const uint32_t raw = smem_u32(dsmem);
  uint8_t* sm = dsmem + ((1024u - (raw & 1023u)) & 1023u);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_pairs = (p.n_q_tiles + 1) / 2;
  // Grid: (unit, clip*head), or (clip*head, unit) under the block-causal mask
  // so that the hardware starts the heaviest units of every head first.  A
  // unit is a pair of query tiles (TILES == 2) or one query tile, later
  // (heavier) tiles first.
  const int unit = p.mask == JEPA_B200_MASK_BLOCK_CAUSAL ? static_cast<int>(blockIdx.y) : static_cast<int>(blockIdx.x);
  const int bh = p.mask == JEPA_B200_MASK_BLOCK_CAUSAL ? static_cast<int>(blockIdx.x) : static_cast<int>(blockIdx.y);
  // The CLS tile (query rows 0..127 against every key, only row 0 kept) is
  // the second tile of the last pair when the tile count is odd (that pair
  // has no second tile of its own), else the one tile of unit 0.
  const int cls_unit = p.cls_separate && !(TILES == 2 ? p.cls_in_pair : p.cls_tail);
  const bool cls_cta = cls_unit && unit == 0;
  int q00, q01 = 0, nkv0, nkv1 = 0, cls_g = cls_cta ? 0 : -1;  // cls_g: query tile g holding CLS
  if (TILES == 2) {
    const int pair = n_pairs - 1 - (unit - cls_unit);
    if (!cls_cta && p.cls_in_pair && pair == n_pairs - 1) cls_g = 1;
    q00 = cls_cta ? 0 : 2 * pair * 128;  // first rows of query tiles 0 and 1
    q01 = cls_g == 1 ? 0 : q00 + 128;
    nkv0 = cls_cta ? (p.N + 127) / 128 : kv_tiles(p, q00);
    nkv1 = cls_cta ? 0 : (cls_g == 1 ? (p.N + 127) / 128 : kv_tiles(p, q01));
  } else {
    q00 = cls_cta ? 0 : (p.n_q_tiles - 1 - (unit - cls_unit)) * 128;
    nkv0 = cls_cta ? (p.N + 127) / 128 : kv_tiles(p, q00);
  }
  // One tile per CTA with N % 128 != 0: the CLS query rides in row N, the
  // first padding row of the last query tile, which visits every KV tile.
  const bool tail_cls = TILES == 1 && p.cls_tail && !cls_cta && q00 == (p.n_q_tiles - 1) * 128;
  const int nkv_all = max(nkv0, nkv1);

  if (threadIdx.x == 0) {
    mbar_init(&q_full, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], TILES);  // one release per MMA issuer
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], TILES);
    }
    for (int g = 0; g < 2; ++g) {
      mbar_init(&s_full[g], 1);
      mbar_init(&s_free[g], 256);
      mbar_init(&p_full[g], 256);
      mbar_init(&pv_done[g], 1);
      mbar_init(&drain_bar[g], 1);
      mbar_init(&x_bar[g], 256);
    }
    mbar_init(&stagger_bar, 256);
    abort_sh = 0;
    mbar_fence_init();
  }
  if (warp == 1) {
    tmem_alloc(&tmem_sh, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_sh;
  pdl_wait();  // Q, K, V^T come from the previous kernel
  pdl_trigger();

  WaitCtl w;
  w.abort = reinterpret_cast<volatile int*>(&abort_sh);
  w.err = p.err;
  w.timeout_ns = p.timeout_ns;
  w.where = (KID_ATTN << 8) | static_cast<unsigned>(warp);

  if (warp == 0) {
    if (lane == 0) {
      bool ok = true;
      uint32_t karmed = 0, kpar = 0, varmed = 0, vpar = 0;
      mbar_expect_tx(&q_full, nkv1 > 0 ? 2 * kTile : kTile);
      tma_load_3d(sm + C::kOffQ, &tmQ, &q_full, 0, q00, bh);
      if (nkv1 > 0) tma_load_3d(sm + C::kOffQ + kTile, &tmQ, &q_full, 0, q01, bh);
      for (int j = 0; j < nkv_all; ++j) {
        const int s = j % kStages;
        const uint32_t ph = (j / kStages) & 1;
        if (!mbar_wait(&k_empty[s], ph ^ 1, w)) {
          ok = false;
          break;
        }
        mbar_expect_tx(&k_full[s], kTile);
        tma_load_3d(sm + C::kOffK + s * kTile, &tmK, &k_full[s], 0, j * 128, bh);
        karmed |= 1u << s;
        kpar = (kpar & ~(1u << s)) | (ph << s);
        if (!mbar_wait(&v_empty[s], ph ^ 1, w)) {
          ok = false;
          break;
        }
        mbar_expect_tx(&v_full[s], kTile);
        tma_load_3d(sm + C::kOffV + s * kTile, &tmV, &v_full[s], j * 128, 0, bh);
        tma_load_3d(sm + C::kOffV + s * kTile + kTile / 2, &tmV, &v_full[s], j * 128 + 64, 0, bh);
        varmed |= 1u << s;
        vpar = (vpar & ~(1u << s)) | (ph << s);
      }
      if (!ok) {  // let the copies already issued land before the CTA exits
        mbar_wait_drain(&q_full, 0);
        for (int s = 0; s < kStages; ++s) {
          if ((karmed >> s) & 1u) mbar_wait_drain(&k_full[s], (kpar >> s) & 1u);
          if ((varmed >> s) & 1u) mbar_wait_drain(&v_full[s], (vpar >> s) & 1u);
        }
      }
    }
  } else if (warp == 1 || (TILES == 2 && warp == 18)) {
    // one MMA issuer per query tile, so each tile's S / PV products follow
    // its own softmax without waiting on the other tile's
    bool okq = true;
    if (tail_cls) {
      // once the Q tile has landed (its rows past N zero-filled), eight lanes
      // write Q[bh, 0, :] into row N - q00 of it in the 128-byte-swizzled
      // layout, then make the writes visible to the tensor core
      okq = __all_sync(0xffffffffu, mbar_wait(&q_full, 0, w));
      if (okq && lane < 8) {
        const uint4 v = *reinterpret_cast<const uint4*>(p.q + static_cast<size_t>(bh) * p.N * 64 + lane * 8);
        st_shared_v4(smem_u32(sm + C::kOffQ) + sw128_offset(p.N - q00, lane * 8), v.x, v.y, v.z, v.w);
      }
      fence_proxy_async_smem();
      __syncwarp();
    }
    if (lane == 0 && okq) {
      const int g = warp == 1 ? 0 : 1;
      const int nkv_g = g == 0 ? nkv0 : nkv1;
      constexpr uint32_t idesc_s = idesc_f16_f32(128, 128, BF);
      constexpr uint32_t idesc_o = idesc_f16_f32(128, 64, BF);
      const uint64_t qd = sdesc_kmajor_sw128(smem_u32(sm + C::kOffQ + g * kTile));
      bool ok = mbar_wait(&q_full, 0, w);
      // Every issuer waits for each K / V tile to land and then arrives on
      // its release barrier (count 2), also for tiles it does not use: a
      // stage is only refilled once both issuers are done with it.
      for (int j = 0; ok && j <= nkv_all; ++j) {
        const int ks = j % kStages;
        if (j < nkv_all) {
          if (!mbar_wait(&k_full[ks], (j / kStages) & 1, w)) {
            ok = false;
            break;
          }
          if (j < nkv_g) {  // S_g = Q_g K_j^T once softmax g has taken S_g of tile j-1
            if (j > 0 && !mbar_wait(&s_free[g], (j - 1) & 1, w)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint64_t kd = sdesc_kmajor_sw128(smem_u32(sm + C::kOffK + ks * kTile));
#pragma unroll
            for (int k = 0; k < 4; ++k)
              tc_mma_f16_ss(tmem + C::kColS + 128 * g, qd + static_cast<uint64_t>(2 * k),
                            kd + static_cast<uint64_t>(2 * k), idesc_s, k > 0 ? 1u : 0u);
            tc_commit(&s_full[g]);
          }
          tc_commit(&k_empty[ks]);
        }
        if (j >= 1) {
          const int vs = (j - 1) % kStages;
          if (!mbar_wait(&v_full[vs], ((j - 1) / kStages) & 1, w)) {
            ok = false;
            break;
          }
          if (j <= nkv_g) {  // O_g += P_g V_{j-1} (P from TMEM) once softmax g published P_g
            if (!mbar_wait(&p_full[g], (j - 1) & 1, w)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t vb = smem_u32(sm + C::kOffV + vs * kTile);
#pragma unroll
            for (int k = 0; k < 8; ++k) {
              const uint64_t bd = sdesc_kmajor_sw128(vb + (k >> 2) * (kTile / 2)) + static_cast<uint64_t>(2 * (k & 3));
              tc_mma_f16_ts(tmem + C::kColO + 64 * g, tmem + C::kColP + 64 * g + 8 * k, bd, idesc_o,
                            (j > 1 || k > 0) ? 1u : 0u);
            }
            tc_commit(&pv_done[g]);
          }
          tc_commit(&v_empty[vs]);
        }
      }
      tc_commit(&drain_bar[g]);
      mbar_wait_drain(&drain_bar[g], 0);
    }
  } else if constexpr (ROWS_IN_WARP) {
    // softmax: warps 2-9 take query tile 0, warps 10-17 query tile 1.  The
    // two warps of a TMEM lane quadrant take its 32 rows in halves of 16;
    // through the 16-lane TMEM shapes four threads share a row, each with 32
    // of a KV tile's 128 keys, and every thread holds two rows (ra, ra + 8),
    // so row maxima and row sums are reduced with two shuffles in the warp.
    const int g = (warp - 2) >> 3;
    const int hh = ((warp - 2) >> 2) & 1;
    const int quad = warp & 3;
    const int lane_base = quad * 32 + hh * 16;
    const int kq = lane & 3;  // this thread's keys in every group of 8: 2*kq, 2*kq + 1
    const int ra = lane_base + (lane >> 2);
    const int q0 = g == 0 ? q00 : q01;
    const int ia = q0 + ra, ib = ia + 8;
    const int n_my = g == 0 ? nkv0 : nkv1;
    const uint32_t lane_off = static_cast<uint32_t>(lane_base) << 16;
    const uint32_t tS = tmem + C::kColS + 128 * g + lane_off;
    const uint32_t tO = tmem + C::kColO + 64 * g + lane_off;
    const uint32_t tP = tmem + C::kColP + 64 * g + lane_off;
    int loa, hia, lob, hib;
    const bool cls_tile = g == cls_g;
    row_keys(p, cls_tile, ia, loa, hia);
    row_keys(p, cls_tile, ib, lob, hib);
    const float c = p.scale_log2;
    float m_a = -INFINITY, m_b = -INFINITY, l_a = 0.0f, l_b = 0.0f;  // l: this thread's share of the row sum
    bool ok = true;
    for (int j = 0; ok && j < n_my; ++j) {
      bool okw = mbar_wait(&s_full[g], j & 1, w);
      okw = __all_sync(0xffffffffu, okw);
      if (!okw) {
        ok = false;
        break;
      }
      tc_fence_after();
      float s[64];
      {
        uint32_t u[64];
        tmem_ld_16x256b_x16(tS, u);
#pragma unroll
        for (int e = 0; e < 64; ++e) s[e] = __uint_as_float(u[e]);
      }
      tc_fence_before();
      mbar_arrive(&s_free[g]);  // S_g may now be overwritten by the next KV tile
      const int kbase = j * 128;
      const bool full = loa <= kbase && hia >= kbase + 127 && lob <= kbase && hib >= kbase + 127;
      if (!__all_sync(0xffffffffu, full)) {
#pragma unroll
        for (int m = 0; m < 16; ++m) {
          const int key = kbase + 8 * m + 2 * kq;
          s[4 * m] = (key >= loa && key <= hia) ? s[4 * m] : -INFINITY;
          s[4 * m + 1] = (key + 1 >= loa && key + 1 <= hia) ? s[4 * m + 1] : -INFINITY;
          s[4 * m + 2] = (key >= lob && key <= hib) ? s[4 * m + 2] : -INFINITY;
          s[4 * m + 3] = (key + 1 >= lob && key + 1 <= hib) ? s[4 * m + 3] : -INFINITY;
        }
      }
      float xa = fmaxf(s[0], s[1]), xb = fmaxf(s[2], s[3]);
      float ya = fmaxf(s[4], s[5]), yb = fmaxf(s[6], s[7]);
#pragma unroll
      for (int m = 2; m < 16; m += 2) {
        xa = fmax3(xa, s[4 * m], s[4 * m + 1]);
        xb = fmax3(xb, s[4 * m + 2], s[4 * m + 3]);
        ya = fmax3(ya, s[4 * m + 4], s[4 * m + 5]);
        yb = fmax3(yb, s[4 * m + 6], s[4 * m + 7]);
      }
      float mxa = fmaxf(xa, ya), mxb = fmaxf(xb, yb);
      mxa = fmaxf(mxa, __shfl_xor_sync(0xffffffffu, mxa, 1));
      mxb = fmaxf(mxb, __shfl_xor_sync(0xffffffffu, mxb, 1));
      mxa = fmaxf(mxa, __shfl_xor_sync(0xffffffffu, mxa, 2));
      mxb = fmaxf(mxb, __shfl_xor_sync(0xffffffffu, mxb, 2));
      const float mna = fmaxf(m_a, mxa * c), mnb = fmaxf(m_b, mxb * c);
      const bool ga = mna > m_a + kRescaleLog2, gb = mnb > m_b + kRescaleLog2;
      const float alpha_a = ga ? ex2_approx(m_a - mna) : 1.0f;  // exp2(-inf) = 0 on the first tile
      const float alpha_b = gb ? ex2_approx(m_b - mnb) : 1.0f;
      l_a *= alpha_a;
      l_b *= alpha_b;
      if (ga) m_a = mna;
      if (gb) m_b = mnb;
      // a row that has seen no allowed key yet keeps m = -inf: all its p are 0
      const float mua = m_a == -INFINITY ? 0.0f : m_a, mub = m_b == -INFINITY ? 0.0f : m_b;
      // P = exp2(s*c - m), two lanes at a time, packed as f16 pairs in the
      // 16x128b order (one word per row and 4-column group); computed
      // before waiting for the previous PV product, which only the O
      // rescale and the P store depend on
      const uint64_t c2 = f2_pack(c, c), nma = f2_pack(-mua, -mua), nmb = f2_pack(-mub, -mub);
      uint64_t sa[2] = {0ull, 0ull}, sb[2] = {0ull, 0ull};
      uint32_t pk[32];
#pragma unroll
      for (int m = 0; m < 16; ++m) {
        float x0, x1, x2, x3;
        f2_unpack(f2_fma(f2_pack(s[4 * m], s[4 * m + 1]), c2, nma), x0, x1);
        f2_unpack(f2_fma(f2_pack(s[4 * m + 2], s[4 * m + 3]), c2, nmb), x2, x3);
        const float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
        const float p2 = ex2_approx(x2), p3 = ex2_approx(x3);
        sa[m & 1] = f2_add(sa[m & 1], f2_pack(p0, p1));
        sb[m & 1] = f2_add(sb[m & 1], f2_pack(p2, p3));
        pk[2 * m] = pack2<BF>(p0, p1);
        pk[2 * m + 1] = pack2<BF>(p2, p3);
      }
      if (j > 0) {  // P_g free and O_g stable once the PV product of tile j-1 is done
        okw = mbar_wait(&pv_done[g], (j - 1) & 1, w);
        okw = __all_sync(0xffffffffu, okw);
        if (!okw) {
          ok = false;
          break;
        }
      }
      tc_fence_after();
      // tcgen05.ld / st are warp-collective: the warp rescales together
      if (j > 0 && __any_sync(0xffffffffu, ga || gb)) {
        uint32_t o[32];
        tmem_ld_16x256b_x8(tO, o);
#pragma unroll
        for (int m = 0; m < 8; ++m) {
          o[4 * m] = __float_as_uint(__uint_as_float(o[4 * m]) * alpha_a);
          o[4 * m + 1] = __float_as_uint(__uint_as_float(o[4 * m + 1]) * alpha_a);
          o[4 * m + 2] = __float_as_uint(__uint_as_float(o[4 * m + 2]) * alpha_b);
          o[4 * m + 3] = __float_as_uint(__uint_as_float(o[4 * m + 3]) * alpha_b);
        }
        tmem_st_16x256b_x8(tO, o);
      }
      tmem_st_16x128b_x16(tP, pk);
      float t0, t1, t2, t3;
      f2_unpack(f2_add(sa[0], sa[1]), t0, t1);
      f2_unpack(f2_add(sb[0], sb[1]), t2, t3);
      l_a += t0 + t1;
      l_b += t2 + t3;
      tc_fence_before();
      mbar_arrive(&p_full[g]);
    }
    if (ok && n_my > 0) {  // the last PV product completes after all earlier ones
      bool okw = mbar_wait(&pv_done[g], (n_my - 1) & 1, w);
      okw = __all_sync(0xffffffffu, okw);
      l_a += __shfl_xor_sync(0xffffffffu, l_a, 1);
      l_b += __shfl_xor_sync(0xffffffffu, l_b, 1);
      l_a += __shfl_xor_sync(0xffffffffu, l_a, 2);
      l_b += __shfl_xor_sync(0xffffffffu, l_b, 2);
      if (okw) {
        tc_fence_after();
        const float inv_a = l_a > 0.0f ? 1.0f / l_a : 0.0f;
        const float inv_b = l_b > 0.0f ? 1.0f / l_b : 0.0f;
        const int b = bh / p.heads, hd = bh % p.heads;
        uint32_t o[32];
        tmem_ld_16x256b_x8(tO, o);
        // rows this CTA writes: the CLS CTA only row 0; pair CTAs every
        // valid row but a separately computed CLS row
        // row N of the last tile holds the CLS query (tail_cls): output row 0
        const bool st_a = cls_tile ? (ia == 0) : ((ia < p.N && !(ia == 0 && p.cls_separate)) || (tail_cls && ia == p.N));
        const bool st_b = cls_tile ? (ib == 0) : ((ib < p.N && !(ib == 0 && p.cls_separate)) || (tail_cls && ib == p.N));
        const int oa = ia == p.N ? 0 : ia, ob = ib == p.N ? 0 : ib;
        // dims 8m + 2kq, 8m + 2kq + 1 of the head; only the first p.dv are written
        if (st_a) {
          uint32_t* dst = reinterpret_cast<uint32_t*>(p.out + (static_cast<size_t>(b) * p.N + oa) * p.ldo + hd * p.dv + 2 * kq);
#pragma unroll
          for (int m = 0; m < 8; ++m)
            if (8 * m < p.dv)
              dst[4 * m] = pack2<BF>(__uint_as_float(o[4 * m]) * inv_a, __uint_as_float(o[4 * m + 1]) * inv_a);
        }
        if (st_b) {
          uint32_t* dst = reinterpret_cast<uint32_t*>(p.out + (static_cast<size_t>(b) * p.N + ob) * p.ldo + hd * p.dv + 2 * kq);
#pragma unroll
          for (int m = 0; m < 8; ++m)
            if (8 * m < p.dv)
              dst[4 * m] = pack2<BF>(__uint_as_float(o[4 * m + 2]) * inv_b, __uint_as_float(o[4 * m + 3]) * inv_b);
        }
      }
    }
  } else {
    // softmax, rows split across warps: warps 2-9 take query tile 0, warps
    // 10-17 query tile 1; two threads per query row (in two warps of the
    // same TMEM lane quadrant), each with half of the 128 keys of a tile
    // (and half of the 64 output columns), row maxima and sums combined
    // through shared memory behind a bounded barrier
    const int g = (warp - 2) >> 3;
    const int ch = ((warp - 2) >> 2) & 1;
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    const int i = (g == 0 ? q00 : q01) + r;
    const int n_my = g == 0 ? nkv0 : nkv1;
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t tS = tmem + C::kColS + 128 * g + 64 * ch + lane_off;
    const uint32_t tO = tmem + C::kColO + 64 * g + 32 * ch + lane_off;
    const uint32_t tP = tmem + C::kColP + 64 * g + 32 * ch + lane_off;
    int lo, hi;
    key_range(p, i, lo, hi);
    const bool cls_tile = g == cls_g;
    if (i >= p.N || cls_tile) {
      lo = 0;
      hi = p.N - 1;
    }
    // rows this CTA writes: the CLS CTA only row 0; pair CTAs every valid row
    // but a separately computed CLS row
    const bool store_row = cls_tile ? (i == 0) : (i < p.N && !(i == 0 && p.cls_separate));
    const float c = p.scale_log2;
    float m_run = -INFINITY, l_run = 0.0f;
    bool ok = true;
    // Stagger: query tile 1 starts once tile 0 has its first P, so that one
    // tile's exponentials overlap the other's TMEM traffic and row-max
    // exchange (these bidirectional tiles are long; the block-causal layout
    // above is faster without it).
    if (g == 1 && nkv0 > 0 && n_my > 0) {
      bool okw = mbar_wait(&stagger_bar, 0, w);
      ok = __all_sync(0xffffffffu, okw);
    }
    for (int j = 0; ok && j < n_my; ++j) {
      bool okw = mbar_wait(&s_full[g], j & 1, w);
      okw = __all_sync(0xffffffffu, okw);
      if (!okw) {
        ok = false;
        break;
      }
      tc_fence_after();
      float s[64];
      {
        uint32_t u[64];
        tmem_ld64(tS, u);
#pragma unroll
        for (int e = 0; e < 64; ++e) s[e] = __uint_as_float(u[e]);
      }
      tc_fence_before();
      mbar_arrive(&s_free[g]);  // S_g may now be overwritten by the next KV tile
      const int kbase = j * 128 + 64 * ch;
      const bool full = lo <= kbase && hi >= kbase + 63;
      if (!__all_sync(0xffffffffu, full)) {
        const int rlo = lo - kbase, rhi = hi - kbase;
#pragma unroll
        for (int e = 0; e < 64; ++e) s[e] = (e >= rlo && e <= rhi) ? s[e] : -INFINITY;
      }
      float mxv[4];
#pragma unroll
      for (int t = 0; t < 4; ++t) mxv[t] = fmax3(s[t], s[4 + t], s[8 + t]);
#pragma unroll
      for (int e = 12; e < 60; e += 8) {
#pragma unroll
        for (int t = 0; t < 4; ++t) mxv[t] = fmax3(mxv[t], s[e + t], s[e + 4 + t]);
      }
#pragma unroll
      for (int t = 0; t < 4; ++t) mxv[t] = fmaxf(mxv[t], s[60 + t]);
      // the other half of the row: exchange partial maxima through shared
      // memory (double-buffered by tile parity; bounded barrier wait)
      xmax[j & 1][g][ch][r] = fmaxf(fmaxf(mxv[0], mxv[1]), fmaxf(mxv[2], mxv[3]));
      mbar_arrive(&x_bar[g]);
      okw = mbar_wait(&x_bar[g], j & 1, w);
      okw = __all_sync(0xffffffffu, okw);
      if (!okw) {
        ok = false;
        break;
      }
      const float mx = fmaxf(xmax[j & 1][g][0][r], xmax[j & 1][g][1][r]);
      const float m_new = fmaxf(m_run, mx * c);
      const bool grow = m_new > m_run + kRescaleLog2;
      const float alpha = grow ? ex2_approx(m_run - m_new) : 1.0f;  // exp2(-inf) = 0 on the first tile
      l_run *= alpha;
      if (grow) m_run = m_new;
      // a row that has seen no allowed key yet keeps m = -inf: all its p are 0
      const float m_use = m_run == -INFINITY ? 0.0f : m_run;
      // P = exp2(s*c - m): arguments and the row sum two lanes at a time,
      // packed as f16 pairs; computed before waiting for the previous PV
      // product, which only the O rescale and the P store depend on
      const uint64_t c2 = f2_pack(c, c), nm2 = f2_pack(-m_use, -m_use);
      uint64_t lsv2[4] = {0ull, 0ull, 0ull, 0ull};
      uint32_t pk[32];
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        float xa, xb;
        f2_unpack(f2_fma(f2_pack(s[2 * e], s[2 * e + 1]), c2, nm2), xa, xb);
        const float pa = ex2_approx(xa);
        const float pb = ex2_approx(xb);
        lsv2[e & 3] = f2_add(lsv2[e & 3], f2_pack(pa, pb));
        pk[e] = pack2<BF>(pa, pb);
      }
      if (j == 0 && g == 0) mbar_arrive(&stagger_bar);
      if (j > 0) {  // P_g free and O_g stable once the PV product of tile j-1 is done
        okw = mbar_wait(&pv_done[g], (j - 1) & 1, w);
        okw = __all_sync(0xffffffffu, okw);
        if (!okw) {
          ok = false;
          break;
        }
      }
      tc_fence_after();
      // tcgen05.ld / st are warp-collective: the warp rescales together
      if (j > 0 && __any_sync(0xffffffffu, grow)) {
#pragma unroll 1
        for (int q = 0; q < 2; ++q) {
          uint32_t o[16];
          tmem_ld16(tO + static_cast<uint32_t>(q * 16), o);
#pragma unroll
          for (int e = 0; e < 16; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
          tmem_st16(tO + static_cast<uint32_t>(q * 16), o);
        }
      }
      tmem_st32(tP, pk);
      float lsv[8];
#pragma unroll
      for (int t = 0; t < 4; ++t) f2_unpack(lsv2[t], lsv[2 * t], lsv[2 * t + 1]);
      l_run += ((lsv[0] + lsv[1]) + (lsv[2] + lsv[3])) + ((lsv[4] + lsv[5]) + (lsv[6] + lsv[7]));
      tc_fence_before();
      mbar_arrive(&p_full[g]);
    }
    if (ok && n_my > 0) {  // the last PV product completes after all earlier ones
      bool okw = mbar_wait(&pv_done[g], (n_my - 1) & 1, w);
      xsum[g][ch][r] = l_run;
      mbar_arrive(&x_bar[g]);
      okw = okw && mbar_wait(&x_bar[g], n_my & 1, w);
      okw = __all_sync(0xffffffffu, okw);
      if (okw) {
        tc_fence_after();
        const float l_row = xsum[g][0][r] + xsum[g][1][r];
        const float inv_l = l_row > 0.0f ? 1.0f / l_row : 0.0f;
        const int b = bh / p.heads, hd = bh % p.heads;
        uint32_t o[32];
        tmem_ld32(tO, o);
        if (store_row && ch * 32 < p.dv) {  // this thread's dims 32ch .. 32ch + 31 of the head
          uint4* dst = reinterpret_cast<uint4*>(p.out + (static_cast<size_t>(b) * p.N + i) * p.ldo + hd * p.dv + ch * 32);
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            uint32_t h[4];
#pragma unroll
            for (int e = 0; e < 4; ++e)
              h[e] = pack2<BF>(__uint_as_float(o[8 * u + 2 * e]) * inv_l, __uint_as_float(o[8 * u + 2 * e + 1]) * inv_l);
            dst[u] = make_uint4(h[0], h[1], h[2], h[3]);
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_sh, C::kTmemCols);
  }
}

int attn_prepare(AttnOp* op, const __half* q, const __half* k, const __half* vt, int B, int heads, int ntok,
                 int npad, int mask, int has_cls, int ppf, __half* out, int head_dim) {
  if (!op || !q || !k || !vt || !out) return JEPA_B200_ERR_ARG;
  if (head_dim != 32 && head_dim != 64) return JEPA_B200_ERR_SHAPE;
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
  // softmax scale 1/sqrt(head_dim) in the exp2 domain; a 32-dim head runs
  // as a 64-dim one whose dims 32..63 are zero in Q, K and V^T
  p.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(head_dim)));
  p.out = out;
  p.dv = head_dim;
  p.ldo = heads * head_dim;
  p.cls_separate = (mask == JEPA_B200_MASK_BLOCK_CAUSAL && has_cls) ? 1 : 0;
  p.cls_in_pair = (p.cls_separate && p.n_q_tiles % 2 == 1) ? 1 : 0;
  p.cls_tail = (p.cls_separate && ntok % 128 != 0) ? 1 : 0;
  p.q = q;
  op->q = q;
  op->k = k;
  op->vt = vt;
  op->npad = npad;
  op->B = B;
  op->smem = AttnCfg<2>::kSmem;
  return JEPA_B200_OK;
}

template <bool ROWS_IN_WARP, int TILES, bool BF>
static int attn_launch_impl(const AttnParams& p, const AttnOp& op, cudaStream_t st) {
  using C = AttnCfg<TILES>;
  auto kern = attn_fwd_kernel<ROWS_IN_WARP, TILES, BF>;
  static std::atomic<unsigned long long> attr_done{0};
  if (!smem_attr_once(attr_done, kern, C::kSmem)) return JEPA_B200_ERR_CUDA;
  const int units = TILES == 2 ? (p.n_q_tiles + 1) / 2 + (p.cls_separate && !p.cls_in_pair ? 1 : 0)
                               : p.n_q_tiles + (p.cls_separate && !p.cls_tail ? 1 : 0);
  const dim3 grid = p.mask == JEPA_B200_MASK_BLOCK_CAUSAL ? dim3(op.B * p.heads, units) : dim3(units, op.B * p.heads);
  if (launch_pdl(kern, grid, dim3(C::kThreads), C::kSmem, st, 1, op.tmQ, op.tmK, op.tmV, p) != cudaSuccess)
    return JEPA_B200_ERR_CUDA;
  return JEPA_B200_OK;
}

// Query tiles per CTA and row layout under each mask.
constexpr int kTilesBlockCausal = 1;
constexpr int kTilesBidir = 2;
constexpr bool kRowsInWarpBlockCausal = true;
constexpr bool kRowsInWarpBidir = false;

int attn_launch(const AttnOp& op, cudaStream_t st, DevErr* err, unsigned long long timeout_ns) {
  AttnParams p = op.p;
  p.err = err;
  p.timeout_ns = timeout_ns;
  // Block-causal query tiles visit few KV tiles, where the per-tile row-max
  // exchange between warps is a large share: rows kept inside one warp.
  // Bidirectional tiles are long and bound by the exponentials, where the
  // cross-warp layout issues fewer instructions.
  if (p.mask == JEPA_B200_MASK_BLOCK_CAUSAL)
    return op.bf16 ? attn_launch_impl<kRowsInWarpBlockCausal, kTilesBlockCausal, true>(p, op, st)
                   : attn_launch_impl<kRowsInWarpBlockCausal, kTilesBlockCausal, false>(p, op, st);
  return op.bf16 ? attn_launch_impl<kRowsInWarpBidir, kTilesBidir, true>(p, op, st)
                 : attn_launch_impl<kRowsInWarpBidir, kTilesBidir, false>(p, op, st);
}

}  // namespace jb
