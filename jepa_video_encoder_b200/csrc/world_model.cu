// The LeWM world model on the GPU: the AdaLN-zero causal predictor and its
// rollout in one kernel ("LeWorldModel Push-T" card, intro: six AdaLN-zero
// causal blocks conditioned on a 10-d action roll the projected CLS state
// forward; benchmarks page, "LeWM world model": one predictor call over a
// 3-frame window of 192-d states, a rollout growing that window one predicted
// state per step).
//
// The work is a few rows (candidates x window frames, at most 32 per CTA)
// against about 4 M weights, so it is bound by streaming the weights, not by
// arithmetic, and a launch per layer would cost more than the layer.  One CTA
// runs every step of a group of candidates:
//   * the weights stream through shared memory as 128-row x 64-column f16
//     tiles (TMA, 128-byte swizzle) and are the M operand of tcgen05.mma; the
//     state rows (32, zero-padded) are the N operand, so an accumulator tile
//     holds 128 output features (TMEM lanes) x 32 rows (columns);
//   * the residual stream x stays in shared memory, transposed (feature-major)
//     and in f32; the four epilogue warps own one feature per TMEM lane and
//     write each phase's result where the next phase reads it (the next B
//     operand, or x);
//   * LayerNorm statistics, the modulation, GELU, the gated residual updates
//     and the causal attention over the window (at most 32 keys) run on CUDA
//     cores in f32;
//   * the adaLN modulation of a block ([shift1 scale1 gate1] and then
//     [shift2 scale2 gate2]) stays in TMEM, each chunk starting at a tile
//     boundary so that feature n of every chunk sits in TMEM lane n % 128.
// Warp roles: 0 TMA producer, 1 MMA issuer (and TMEM owner), 2-5 epilogue.
#include <algorithm>

#include "internal.h"
#include "world_model.h"

namespace jb {
namespace {

constexpr int kR = 32;             // state rows per CTA (the MMA's N)
constexpr int kStages = 6;         // weight tiles in flight
constexpr int kTile = 16384;       // 128 rows x 64 f16
constexpr int kThreads = 192;
constexpr int kTmemCols = 512;
constexpr int kColMod = 0;         // adaLN chunks: 3 x ceil(D/128) tiles of 32 columns
constexpr int kColAcc = 192;       // accumulators: up to 10 tiles
constexpr int kXLd = kR + 1;       // f32 per feature row of the transposed x
constexpr int kQLd = kR + 2;       // 16-bit values per feature row of the transposed q|k|v
constexpr int kHeadDim = 64;
constexpr float kQkScale = 0.125f;  // 1 / sqrt(kHeadDim)

enum : int { ARENA_D = 0, ARENA_M = 1, ARENA_H = 2 };
enum : int { BUF_H = 0, BUF_S = 1, BUF_U = 2 };

struct Layout {
  uint32_t hbuf, sbuf, ubuf, xt, stats, bars, total;
};

__host__ __device__ inline Layout wm_layout(int D, int mlp, int hq) {
  Layout s;
  uint32_t o = kStages * kTile;
  s.hbuf = o;
  o += static_cast<uint32_t>(D / 64) * (kR * 128);
  s.sbuf = o;
  o += static_cast<uint32_t>(D / 64) * (kR * 128);
  s.ubuf = o;
  const uint32_t ub = static_cast<uint32_t>((mlp > hq ? mlp : hq) / 64) * (kR * 128);
  const uint32_t qb = static_cast<uint32_t>(3 * D) * kQLd * 2;
  o += ((ub > qb ? ub : qb) + 1023u) / 1024u * 1024u;
  s.xt = o;
  o += static_cast<uint32_t>(D) * kXLd * 4;
  s.stats = o;
  o += 2 * kR * 4;
  s.bars = (o + 7u) / 8u * 8u;
  o = s.bars + (2 * kStages + 3) * 8 + 16;
  s.total = o;
  return s;
}

// One MMA phase: ntiles accumulator tiles of 128 output features, each over
// kchunks 64-wide K chunks.  Tile t reads weight rows row0 + (t / tpc) * crows
// + 128 * (t % tpc) of its arena (tpc tiles per chunk of crows rows).
struct Phase {
  int arena, row0, ntiles, tpc, crows, kchunks, buf, col;
};

__device__ __forceinline__ Phase wm_phase(const WmParams& p, int i) {
  const int D = p.D, Tc = (D + 127) / 128, kD = D / 64;
  const int blk = 10 * D + p.mlp;  // arena-D rows of a block: adaLN, qkv, out, up
  if (i == 0) return {ARENA_D, 0, Tc, Tc, 0, kD, BUF_H, kColAcc};  // action_embed.2
  i -= 1;
  if (i < 6 * p.depth) {
    const int b = i / 6, base = D + b * blk;
    switch (i % 6) {
      case 0: return {ARENA_D, base, 3 * Tc, Tc, D, kD, BUF_S, kColMod};               // adaLN 1st half
      case 1: return {ARENA_D, base + 6 * D, (3 * D + 127) / 128, 1 << 20, 0, kD, BUF_H, kColAcc};  // qkv
      case 2: return {ARENA_D, base + 9 * D, Tc, 1 << 20, 0, kD, BUF_H, kColAcc};       // out
      case 3: return {ARENA_D, base + 3 * D, 3 * Tc, Tc, D, kD, BUF_S, kColMod};       // adaLN 2nd half
      case 4: return {ARENA_D, base + 10 * D, (p.mlp + 127) / 128, 1 << 20, 0, kD, BUF_H, kColAcc};  // up
      default: return {ARENA_M, b * D, Tc, 1 << 20, 0, p.mlp / 64, BUF_U, kColAcc};    // down
    }
  }
  i -= 6 * p.depth;
  if (i == 0) return {ARENA_D, D + p.depth * blk, (p.hq + 127) / 128, 1 << 20, 0, kD, BUF_H, kColAcc};  // proj.0
  return {ARENA_H, 0, Tc, 1 << 20, 0, p.hq / 64, BUF_U, kColAcc};                       // proj.2
}

__device__ __forceinline__ int tile_row(const Phase& ph, int t) {
  return ph.row0 + (t / ph.tpc) * ph.crows + 128 * (t % ph.tpc);
}

// Byte offset of (row r, column k) in a B-operand buffer: K chunks of 64
// columns, each 32 rows x 128 bytes with the 128-byte swizzle.
__device__ __forceinline__ uint32_t boff(int r, int k) {
  return static_cast<uint32_t>(k >> 6) * (kR * 128) + sw128_offset(r, k & 63);
}

__device__ __forceinline__ void feat_sync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }
// Barrier of the four epilogue warps that also ANDs a flag over them.
__device__ __forceinline__ bool feat_all(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, 1, 128, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(v))
      : "memory");
  return r != 0;
}

__device__ __forceinline__ float silu(float x) { return x / (1.0f + expf(-x)); }

template <bool BF>
__device__ __forceinline__ void st16(uint8_t* buf, int r, int k, float v) {
  *reinterpret_cast<unsigned short*>(buf + boff(r, k)) = pack1<BF>(v);
}

template <bool BF>
__global__ void __launch_bounds__(kThreads, 1)
    wm_kernel(const __grid_constant__ CUtensorMap tmD, const __grid_constant__ CUtensorMap tmM,
              const __grid_constant__ CUtensorMap tmH, const WmParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const Layout L = wm_layout(p.D, p.mlp, p.hq);
  uint8_t* ring = smem;
  uint8_t* hbuf = smem + L.hbuf;
  uint8_t* sbuf = smem + L.sbuf;
  uint8_t* ubuf = smem + L.ubuf;
  unsigned short* qkv = reinterpret_cast<unsigned short*>(smem + L.ubuf);  // aliases ubuf (dead in between)
  float* xt = reinterpret_cast<float*>(smem + L.xt);
  float* st_mean = reinterpret_cast<float*>(smem + L.stats);
  float* st_rstd = st_mean + kR;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.bars);
  uint64_t* empty = full + kStages;
  uint64_t* go_bar = empty + kStages;
  uint64_t* acc_bar = go_bar + 1;
  uint64_t* drain_bar = acc_bar + 1;
  uint32_t* tmem_sh = reinterpret_cast<uint32_t*>(drain_bar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_sh + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int D = p.D, Tc = (D + 127) / 128;
  const int steps = p.steps > 0 ? p.steps : 1;
  const int P = 3 + 6 * p.depth;  // phases per step
  const int c0 = blockIdx.x * p.cpc;
  const int ncl = min(p.cpc, p.n_cand - c0);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(go_bar, 1);
    mbar_init(acc_bar, 1);
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_sh, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_sh;
  WaitCtl w{abort_flag, p.err, p.timeout_ns, (KID_MISC << 8) | static_cast<unsigned>(warp)};
  pdl_wait();

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tmD);
      tma_prefetch_desc(&tmM);
      tma_prefetch_desc(&tmH);
      uint32_t it = 0;
      bool ok = true;
      for (int s = 0; ok && s < steps; ++s)
        for (int i = 0; ok && i < P; ++i) {
          const Phase ph = wm_phase(p, i);
          const CUtensorMap* tm = ph.arena == ARENA_D ? &tmD : (ph.arena == ARENA_M ? &tmM : &tmH);
          for (int t = 0; ok && t < ph.ntiles; ++t)
            for (int kc = 0; kc < ph.kchunks; ++kc, ++it) {
              const uint32_t slot = it % kStages;
              if (it >= kStages && !mbar_wait(&empty[slot], ((it / kStages) - 1) & 1, w)) {
                ok = false;
                break;
              }
              mbar_expect_tx(&full[slot], kTile);
              tma_load_2d(ring + slot * kTile, tm, &full[slot], kc * 64, tile_row(ph, t));
            }
        }
      // every load issued has landed before the CTA may exit
      const uint32_t n = it < kStages ? it : kStages;
      for (uint32_t j = 0; j < n; ++j) {
        const uint32_t k = it - 1 - j;
        mbar_wait_drain(&full[k % kStages], (k / kStages) & 1);
      }
    }
  } else if (warp == 1) {
    // ----------------------------------------------------------- MMA issue
    if (lane == 0) {
      const uint32_t idesc = idesc_f16_f32(128, kR, BF);
      uint32_t it = 0, phase_no = 0;
      bool ok = true;
      for (int s = 0; ok && s < steps; ++s)
        for (int i = 0; ok && i < P; ++i, ++phase_no) {
          const Phase ph = wm_phase(p, i);
          if (!mbar_wait(go_bar, phase_no & 1, w)) {
            ok = false;
            break;
          }
          tc_fence_after();
          uint8_t* bsrc = ph.buf == BUF_H ? hbuf : (ph.buf == BUF_S ? sbuf : ubuf);
          for (int t = 0; ok && t < ph.ntiles; ++t) {
            const uint32_t d = tmem + static_cast<uint32_t>(ph.col + 32 * t);
            for (int kc = 0; kc < ph.kchunks; ++kc, ++it) {
              const uint32_t slot = it % kStages;
              if (!mbar_wait(&full[slot], (it / kStages) & 1, w)) {
                ok = false;
                break;
              }
              tc_fence_after();
              const uint64_t ad = sdesc_kmajor_sw128(smem_u32(ring + slot * kTile));
              const uint64_t bd = sdesc_kmajor_sw128(smem_u32(bsrc + kc * (kR * 128)));
#pragma unroll
              for (int k16 = 0; k16 < 4; ++k16)
                tc_mma_f16_ss(d, ad + 2 * k16, bd + 2 * k16, idesc, (kc | k16) != 0);
              tc_commit(&empty[slot]);
            }
          }
          tc_commit(acc_bar);
        }
      // every MMA issued has completed before TMEM is released
      tc_commit(drain_bar);
      mbar_wait_drain(drain_bar, 0);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;                 // TMEM lane quadrant of this warp
    const int ft = 32 * q + lane;           // feature lane 0..127
    const uint32_t tl = tmem + (static_cast<uint32_t>(32 * q) << 16);
    uint32_t go_no = 0, acc_no = 0;
    bool ok = true;
    auto go = [&]() {
      fence_proxy_async_smem();
      tc_fence_before();
      feat_sync();
      if (ft == 0) mbar_arrive(go_bar);
      ++go_no;
    };
    auto wait_acc = [&]() -> bool {
      bool okw = mbar_wait(acc_bar, acc_no & 1, w);
      ++acc_no;
      okw = feat_all(okw);
      tc_fence_after();
      return okw;
    };
    // row statistics of x over the D features (rows < R): four threads a row
    auto ln_stats = [&](int R) {
      feat_sync();  // x complete
      const int r = ft >> 2, part = ft & 3, n0 = part * (D / 4), n1 = n0 + D / 4;
      float s = 0.0f;
      if (r < R)
        for (int n = n0; n < n1; ++n) s += xt[n * kXLd + r];
      s += __shfl_xor_sync(0xffffffffu, s, 1);
      s += __shfl_xor_sync(0xffffffffu, s, 2);
      const float mean = s / static_cast<float>(D);
      float v = 0.0f;
      if (r < R)
        for (int n = n0; n < n1; ++n) {
          const float d = xt[n * kXLd + r] - mean;
          v = fmaf(d, d, v);
        }
      v += __shfl_xor_sync(0xffffffffu, v, 1);
      v += __shfl_xor_sync(0xffffffffu, v, 2);
      if (part == 0 && r < R) {
        st_mean[r] = mean;
        st_rstd[r] = rsqrtf(v / static_cast<float>(D) + p.eps);
      }
      feat_sync();
    };
    // B operand = LN(x) (1 + scale) + shift, shift / scale the adaLN chunks
    // 0 / 1 in TMEM plus their biases
    auto build_modulated = [&](int R, const float* b_shift, const float* b_scale) {
      for (int t = 0; t < Tc; ++t) {
        const int n = 128 * t + ft;
        uint32_t sh[32], sc[32];
        tmem_ld32(tl + static_cast<uint32_t>(kColMod + 32 * t), sh);
        tmem_ld32(tl + static_cast<uint32_t>(kColMod + 32 * (Tc + t)), sc);
        if (n < D) {
          const float bsh = b_shift[n], bsc = b_scale[n];
#pragma unroll
          for (int r = 0; r < kR; ++r) {
            if (r >= R) break;
            const float y = (xt[n * kXLd + r] - st_mean[r]) * st_rstd[r];
            st16<BF>(hbuf, r, n, fmaf(y, 1.0f + (__uint_as_float(sc[r]) + bsc), __uint_as_float(sh[r]) + bsh));
          }
        }
      }
    };
    // x += gate * (acc + bias), gate the adaLN chunk 2 in TMEM plus its bias
    auto gated_residual = [&](int R, const float* bias, const float* b_gate) {
      for (int t = 0; t < Tc; ++t) {
        const int n = 128 * t + ft;
        uint32_t a[32], g[32];
        tmem_ld32(tl + static_cast<uint32_t>(kColAcc + 32 * t), a);
        tmem_ld32(tl + static_cast<uint32_t>(kColMod + 32 * (2 * Tc + t)), g);
        if (n < D) {
          const float b = bias[n], bg = b_gate[n];
#pragma unroll
          for (int r = 0; r < kR; ++r) {
            if (r >= R) break;
            xt[n * kXLd + r] = fmaf(__uint_as_float(g[r]) + bg, __uint_as_float(a[r]) + b, xt[n * kXLd + r]);
          }
        }
      }
    };
    // ubuf = GELU(acc + bias) over `width` features
    auto gelu_to_u = [&](int R, int width, const float* bias) {
      for (int t = 0; t < (width + 127) / 128; ++t) {
        const int n = 128 * t + ft;
        uint32_t a[32];
        tmem_ld32(tl + static_cast<uint32_t>(kColAcc + 32 * t), a);
        if (n < width) {
          const float b = bias[n];
#pragma unroll
          for (int r = 0; r < kR; ++r) {
            if (r >= R) break;
            st16<BF>(ubuf, r, n, gelu1(__uint_as_float(a[r]) + b));
          }
        }
      }
    };

    for (int s = 0; ok && s < steps; ++s) {
      // the window of this step: frames [lo, nf) of every candidate
      const int nf = p.steps > 0 ? p.T0 + s : p.T0;
      const int lo = nf > p.window ? nf - p.window : 0;
      const int T = nf - lo, R = ncl * T;
      // x = state + pos; B operand = SiLU(action_embed.0(a)) on CUDA cores
      for (int n = ft; n < D; n += 128) {
        for (int r = 0; r < R; ++r) {
          const int cl = r / T, t = r % T, f = lo + t, c = c0 + cl;
          const float sv = f < p.T0 ? p.states[(static_cast<size_t>(c) * p.T0 + f) * D + n]
                                    : p.out[(static_cast<size_t>(c) * p.steps + (f - p.T0)) * D + n];
          xt[n * kXLd + r] = sv + p.pos[t * D + n];
          const float* a = p.actions + (static_cast<size_t>(c) * p.n_act + f) * p.A;
          const float* wr = p.w_act0 + static_cast<size_t>(n) * p.A;
          float h = p.b_act0[n];
          for (int j = 0; j < p.A; ++j) h = fmaf(wr[j], a[j], h);
          st16<BF>(hbuf, r, n, silu(h));
        }
      }
      go();  // action_embed.2
      if (!(ok = wait_acc())) break;
      for (int t = 0; t < Tc; ++t) {  // adaLN input SiLU(c), c = action_embed.2(.) + bias
        const int n = 128 * t + ft;
        uint32_t a[32];
        tmem_ld32(tl + static_cast<uint32_t>(kColAcc + 32 * t), a);
        if (n < D) {
          const float b = p.b_act2[n];
#pragma unroll
          for (int r = 0; r < kR; ++r) {
            if (r >= R) break;
            st16<BF>(sbuf, r, n, silu(__uint_as_float(a[r]) + b));
          }
        }
      }
      for (int b = 0; ok && b < p.depth; ++b) {
        const float* b_qkv = p.b_qkv + static_cast<size_t>(b) * 3 * D;
        const float* b_ada = p.b_ada + static_cast<size_t>(b) * 6 * D;  // [shift1 scale1 gate1 shift2 scale2 gate2]
        go();  // adaLN 1st half -> TMEM
        if (!(ok = wait_acc())) break;
        ln_stats(R);
        build_modulated(R, b_ada, b_ada + D);
        go();  // qkv
        if (!(ok = wait_acc())) break;
        for (int t = 0; t < (3 * D + 127) / 128; ++t) {
          const int n = 128 * t + ft;
          uint32_t a[32];
          tmem_ld32(tl + static_cast<uint32_t>(kColAcc + 32 * t), a);
          if (n < 3 * D) {
            const float b = b_qkv[n];
#pragma unroll
            for (int r = 0; r < kR; ++r) {
              if (r >= R) break;
              qkv[n * kQLd + r] = pack1<BF>(__uint_as_float(a[r]) + b);
            }
          }
        }
        feat_sync();
        // causal attention over the candidate's frames: one thread per (row, head)
        for (int u = ft; u < R * p.heads; u += 128) {
          const int r = u / p.heads, hd = u % p.heads, t = r % T, r0 = r - t;
          const unsigned short* qh = qkv + static_cast<size_t>(hd * kHeadDim) * kQLd;
          const unsigned short* kh = qh + static_cast<size_t>(D) * kQLd;
          const unsigned short* vh = kh + static_cast<size_t>(D) * kQLd;
          float qv[kHeadDim], o[kHeadDim];
#pragma unroll
          for (int d = 0; d < kHeadDim; ++d) {
            qv[d] = widen1<BF>(qh[d * kQLd + r]) * kQkScale;
            o[d] = 0.0f;
          }
          float m = -INFINITY, l = 0.0f;
          for (int j = 0; j <= t; ++j) {
            float sc = 0.0f;
#pragma unroll
            for (int d = 0; d < kHeadDim; ++d) sc = fmaf(qv[d], widen1<BF>(kh[d * kQLd + r0 + j]), sc);
            const float mn = fmaxf(m, sc), al = expf(m - mn), pj = expf(sc - mn);
            l = fmaf(l, al, pj);
#pragma unroll
            for (int d = 0; d < kHeadDim; ++d) o[d] = fmaf(o[d], al, pj * widen1<BF>(vh[d * kQLd + r0 + j]));
            m = mn;
          }
          const float il = 1.0f / l;
#pragma unroll
          for (int d = 0; d < kHeadDim; ++d) st16<BF>(hbuf, r, hd * kHeadDim + d, o[d] * il);
        }
        go();  // out
        if (!(ok = wait_acc())) break;
        gated_residual(R, p.b_out + static_cast<size_t>(b) * D, b_ada + 2 * D);
        go();  // adaLN 2nd half -> TMEM
        if (!(ok = wait_acc())) break;
        ln_stats(R);
        build_modulated(R, b_ada + 3 * D, b_ada + 4 * D);
        go();  // up
        if (!(ok = wait_acc())) break;
        gelu_to_u(R, p.mlp, p.b_up + static_cast<size_t>(b) * p.mlp);
        go();  // down
        if (!(ok = wait_acc())) break;
        gated_residual(R, p.b_down + static_cast<size_t>(b) * D, b_ada + 5 * D);
      }
      if (!ok) break;
      // pred.norm (affine) -> pred.proj.0 -> GELU -> pred.proj.2
      ln_stats(R);
      for (int n = ft; n < D; n += 128) {
        const float g = p.norm_g[n], bb = p.norm_b[n];
        for (int r = 0; r < R; ++r) st16<BF>(hbuf, r, n, fmaf((xt[n * kXLd + r] - st_mean[r]) * st_rstd[r], g, bb));
      }
      go();  // proj.0
      if (!(ok = wait_acc())) break;
      gelu_to_u(R, p.hq, p.b_p0);
      go();  // proj.2
      if (!(ok = wait_acc())) break;
      for (int t = 0; t < Tc; ++t) {
        const int n = 128 * t + ft;
        uint32_t a[32];
        tmem_ld32(tl + static_cast<uint32_t>(kColAcc + 32 * t), a);
        if (n < D) {
          const float b = p.b_p2[n];
#pragma unroll
          for (int r = 0; r < kR; ++r) {
            if (r >= R) break;
            const int cl = r / T, t2 = r % T, c = c0 + cl;
            const float y = __uint_as_float(a[r]) + b;
            if (p.steps == 0)
              p.out[(static_cast<size_t>(c) * p.T0 + t2) * D + n] = y;
            else if (t2 == T - 1)
              p.out[(static_cast<size_t>(c) * p.steps + s) * D + n] = y;
          }
        }
      }
      __threadfence_block();
      feat_sync();  // the next step reads this step's predictions back
    }
  }
  // the MMA warp's last commit covers every MMA it issued
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace

size_t wm_smem_bytes(int D, int mlp, int hq) { return wm_layout(D, mlp, hq).total + 1024; }

int wm_launch(const WmArena& a, const WmParams& prm, cudaStream_t st) {
  WmParams p = prm;
  if (p.D % 64 || p.D < 64 || p.D > 256 || p.D != kHeadDim * p.heads) return JEPA_B200_ERR_SHAPE;
  if (p.mlp % 64 || p.mlp < 64 || p.mlp > 1024 || p.hq % 64 || p.hq < 64 || p.hq > 1024) return JEPA_B200_ERR_SHAPE;
  if (p.window < 1 || p.window > kR || p.A < 1 || p.T0 < 1 || p.steps < 0 || p.n_cand < 1) return JEPA_B200_ERR_SHAPE;
  const int tmax = p.steps > 0 ? std::min(p.window, p.T0 + p.steps - 1) : p.T0;
  if (tmax > p.window || tmax < 1) return JEPA_B200_ERR_SHAPE;
  p.cpc = kR / tmax;
  const size_t smem = wm_smem_bytes(p.D, p.mlp, p.hq);
  auto kern = a.bf16 ? wm_kernel<true> : wm_kernel<false>;
  // the limit is raised once, to what the largest accepted shape needs
  static std::atomic<unsigned long long> attr_done[2] = {};
  static const int smem_max = static_cast<int>(wm_smem_bytes(256, 1024, 1024));
  if (smem > static_cast<size_t>(smem_max)) return JEPA_B200_ERR_SHAPE;
  if (!smem_attr_once(attr_done[a.bf16 ? 1 : 0], kern, smem_max)) return JEPA_B200_ERR_CUDA;
  const int grid = (p.n_cand + p.cpc - 1) / p.cpc;
  if (launch_pdl(kern, dim3(grid), dim3(kThreads), smem, st, 1, a.tmD, a.tmM, a.tmH, p) != cudaSuccess)
    return JEPA_B200_ERR_CUDA;
  return JEPA_B200_OK;
}

int wm_arena_maps(WmArena* a) {
  if (!make_tmap_2d(&a->tmD, a->d, 2, a->D, a->rows_d, static_cast<uint64_t>(a->D) * 2, 64, 128)) return JEPA_B200_ERR_CUDA;
  if (!make_tmap_2d(&a->tmM, a->m, 2, a->mlp, a->rows_m, static_cast<uint64_t>(a->mlp) * 2, 64, 128))
    return JEPA_B200_ERR_CUDA;
  if (!make_tmap_2d(&a->tmH, a->h, 2, a->hq, a->rows_h, static_cast<uint64_t>(a->hq) * 2, 64, 128))
    return JEPA_B200_ERR_CUDA;
  return JEPA_B200_OK;
}

}  // namespace jb
