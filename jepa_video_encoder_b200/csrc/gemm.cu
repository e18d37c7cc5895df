// tcgen05 GEMM for the encoder's dense layers: out = epilogue(A W^T + bias).
//
// The pre-LN block of the JEPA encoders ("Quantization" page, section "The
// rule": attn_qkv, attn_out, ffn_up, ffn_down per block) spends its time in
// four GEMMs whose A operand is the token matrix [B*N, D] (or [B*N, 4D]) and
// whose B operand is a weight matrix [N_out, K] in PyTorch [out, in] order.
// The tubelet patch-embed (a conv with stride = kernel) is the same GEMM over
// the unfolded patch matrix (built by launch_patchify), with an epilogue that
// adds the positional row and writes the token rows.
//
// Design (one CTA per SM, persistent over output tiles):
//   warp 0      TMA producer: A tile [128 x 64] and, for f16 weights, the
//               B tile [BN x 64] per stage, 128-byte swizzled, into a ring
//               of shared-memory stages;
//   warp 1      MMA issuer: tcgen05.mma kind::f16 M=128 N=BN K=16, f32
//               accumulators in TMEM, two accumulator buffers so the
//               epilogue of tile i overlaps the main loop of tile i+1;
//   warps 2-9   epilogue: tcgen05.ld of the accumulator rows (two warps per
//               TMEM lane quadrant, each half of the columns), bias, then
//               f16 store / GELU / f32 residual add / QKV head scatter /
//               patch-embed + pos_embed;
//   warps 10-13 (quantised weights only) converters: unpack q8_0 (q*d) or
//               q4_0 ((q-8)*d) blocks into the swizzled B tile in shared
//               memory.
// That single-CTA kernel serves the GEMMs of fewer than 256 rows.  The encoder's GEMMs (256 rows or more, f16 weights or the f16 copy
// of dequantised ones) run the CTA-pair variant further down: two SMs share
// a 256 x BN tile through tcgen05.mma.cta_group::2.
#include <cudaTypedefs.h>
#include <string.h>

#include <algorithm>

#include "internal.h"

namespace jb {

template <int BN>
struct GemmCfg {
  static constexpr int BM = 128, BK = 64;
  static constexpr int A_BYTES = BM * BK * 2;
  static constexpr int B_BYTES = BN * BK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int STAGES = BN == 256 ? 4 : (BN == 192 ? 4 : 6);
  static constexpr int TMEM_COLS = 2 * BN <= 256 ? 256 : 512;
  static constexpr int SMEM = STAGES * STAGE_BYTES + 8 * 4096 + 1024;  // + epilogue staging
};

// gelu_q's coefficients, each twice, as the operand pairs of the packed
// polynomial in constant memory: the 128-register kernels read them from the
// constant bank instead of holding twelve register pairs (the same
// coefficients as gelu_q, which a host test compares).
__constant__ float2 kGeluPairs[12] = {
    {-1.000000000e+00f, -1.000000000e+00f}, {-1.151105762e+00f, -1.151105762e+00f},
    {-4.592085183e-01f, -4.592085183e-01f}, {-5.247146264e-02f, -5.247146264e-02f},
    {6.975546945e-03f, 6.975546945e-03f}, {-5.228150712e-06f, -5.228150712e-06f},
    {-2.895472280e-04f, -2.895472280e-04f}, {8.469620661e-05f, 8.469620661e-05f},
    {-1.389817317e-05f, -1.389817317e-05f}, {1.411672088e-06f, 1.411672088e-06f},
    {-8.283102204e-08f, -8.283102204e-08f}, {2.152039880e-09f, 2.152039880e-09f},
};

// Two GELUs in packed f32x2 arithmetic with the coefficient pairs from
// constant memory: the same f32 operations as gelu2 (and gelu1), so the
// same results.
__device__ __forceinline__ void gelu2_cbank(float& x0, float& x1) {
  const float u0 = fabsf(x0), u1 = fabsf(x1);
  const uint64_t c = f2_pack(fminf(u0, 6.0f), fminf(u1, 6.0f));
  uint64_t q = *reinterpret_cast<const uint64_t*>(&kGeluPairs[11]);
#pragma unroll
  for (int k = 10; k >= 0; --k) q = f2_fma(q, c, *reinterpret_cast<const uint64_t*>(&kGeluPairs[k]));
  float q0, q1;
  f2_unpack(q, q0, q1);
  x0 = fmaf(-u0, ex2_approx(q0), fmaxf(x0, 0.0f));
  x1 = fmaf(-u1, ex2_approx(q1), fmaxf(x1, 0.0f));
}

// Two GELUs: coefficient pairs in registers, or (LOWREG, kernels launched
// with 448 threads and so at most 128 registers a thread) in constant
// memory.  The scalar form with immediate coefficients (gelu1) issues twice
// the polynomial's instructions, which in the quantised-weight kernels the
// converter warps on the same SM sub-partitions pay for.
template <bool LOWREG>
__device__ __forceinline__ void gelu_pair(float& a, float& b) {
  if (LOWREG)
    gelu2_cbank(a, b);
  else
    gelu2(a, b);
}

// Rotary positions: turn the pair (x0, x1) at head dims (d, d + 1), d even,
// of the token at (slot, patch row, patch column) = (pt, py, px): axis group
// a = d / 20, pair i = (d % 20) / 2, angle pos_a * 10000^(-2i/20) read from
// the (cos, sin) table; dims 60..63 are not turned.
__device__ __forceinline__ void rope_pair(float& x0, float& x1, int d, int pt, int py, int px, const float2* tab) {
  if (d >= 60) return;
  const int a = d / 20, i = (d - 20 * a) >> 1;
  const int pos = a == 0 ? pt : (a == 1 ? py : px);
  const float2 cs = __ldg(tab + (a * kRopeMaxPos + pos) * 10 + i);
  const float y0 = x0 * cs.x - x1 * cs.y;
  x1 = x0 * cs.y + x1 * cs.x;
  x0 = y0;
}

// The token position of tile row `row` (rows are b * ntok + t, no CLS row).
__device__ __forceinline__ void rope_position(const QkvDst& q, int row, int& pt, int& py, int& px) {
  const int t = row % q.ntok;
  pt = t / q.rope_ppf;
  const int rem = t - pt * q.rope_ppf;
  py = rem / q.rope_pw;
  px = rem - py * q.rope_pw;
}

// Epilogue for 32 consecutive output columns col0..col0+31 of one row.
template <bool LOWREG, bool ROPE, bool BF>
__device__ __forceinline__ void epilogue_chunk(const GemmParams& p, int row, int col0, const uint32_t (&r)[32]) {
  float v[32];
#pragma unroll
  for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
  if (p.bias) {
    const float4* b4 = reinterpret_cast<const float4*>(p.bias + col0);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float4 b = __ldg(b4 + j);
      v[4 * j] += b.x;
      v[4 * j + 1] += b.y;
      v[4 * j + 2] += b.z;
      v[4 * j + 3] += b.w;
    }
  }
  switch (p.epi) {
    case EPI_GELU_F16:
#pragma unroll
      for (int j = 0; j < 16; ++j) gelu_pair<LOWREG>(v[2 * j], v[2 * j + 1]);
      // fall through
    case EPI_F16: {
      uint4* dst = reinterpret_cast<uint4*>(static_cast<__half*>(p.out) + static_cast<size_t>(row) * p.ldo + col0);
#pragma unroll
      for (int j = 0; j < 4; ++j)
        dst[j] = make_uint4(pack2<BF>(v[8 * j], v[8 * j + 1]), pack2<BF>(v[8 * j + 2], v[8 * j + 3]),
                            pack2<BF>(v[8 * j + 4], v[8 * j + 5]), pack2<BF>(v[8 * j + 6], v[8 * j + 7]));
    } break;
    case EPI_RESID_F32: {
      float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.out) + static_cast<size_t>(row) * p.ldo + col0);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        float4 o = dst[j];
        o.x += v[4 * j];
        o.y += v[4 * j + 1];
        o.z += v[4 * j + 2];
        o.w += v[4 * j + 3];
        dst[j] = o;
      }
    } break;
    case EPI_F32: {
      float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.out) + static_cast<size_t>(row) * p.ldo + col0);
#pragma unroll
      for (int j = 0; j < 8; ++j) dst[j] = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
    } break;
    case EPI_QKV: {
      const int D = p.qkv.dim;
      const int part = col0 / D + p.qkv.first_part;
      const int within = col0 % D;
      // head hd of head_dim dims (32 or 64); its values go to dims d0.. of
      // a 64-dim row (with 32-dim heads, dims 32..63 stay zero)
      const int hd = within / p.qkv.head_dim, d0 = within % p.qkv.head_dim;
      const int b = row / p.qkv.ntok, t = row % p.qkv.ntok;
      const size_t bh = static_cast<size_t>(b) * p.qkv.heads + hd;
      if (ROPE && part < 2) {
        int pt, py, px;
        rope_position(p.qkv, row, pt, py, px);
#pragma unroll
        for (int j = 0; j < 16; ++j) rope_pair(v[2 * j], v[2 * j + 1], d0 + 2 * j, pt, py, px, p.qkv.rope);
      }
      if (part < 2) {
        __half* base = part == 0 ? p.qkv.q : p.qkv.k;
        if (base) {
          uint4* dst = reinterpret_cast<uint4*>(base + (bh * p.qkv.ntok + t) * 64 + d0);
#pragma unroll
          for (int j = 0; j < 4; ++j)
            dst[j] = make_uint4(pack2<BF>(v[8 * j], v[8 * j + 1]), pack2<BF>(v[8 * j + 2], v[8 * j + 3]),
                                pack2<BF>(v[8 * j + 4], v[8 * j + 5]), pack2<BF>(v[8 * j + 6], v[8 * j + 7]));
        }
      } else if (p.qkv.vt) {
        __half* base = p.qkv.vt + (bh * 64 + d0) * static_cast<size_t>(p.qkv.npad) + t;
#pragma unroll
        for (int j = 0; j < 32; ++j) base[static_cast<size_t>(j) * p.qkv.npad] = __ushort_as_half(pack1<BF>(v[j]));
      }
    } break;
    case EPI_PATCH: {
      const int b = row / p.patch.n_patches, i = row % p.patch.n_patches;
      const int tok = i + p.patch.has_cls;
      float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.out) +
                                              (static_cast<size_t>(b) * p.patch.ntok + tok) * p.ldo + col0);
      const float4* pos = reinterpret_cast<const float4*>(p.patch.pos + static_cast<size_t>(tok) * p.ldo + col0);
#pragma unroll
      for (int j = 0; j < 8; ++j) {  // a rotary model has no positional table
        const float4 q = p.patch.pos ? __ldg(pos + j) : make_float4(0.f, 0.f, 0.f, 0.f);
        dst[j] = make_float4(v[4 * j] + q.x, v[4 * j + 1] + q.y, v[4 * j + 2] + q.z, v[4 * j + 3] + q.w);
      }
    } break;
    default:
      break;
  }
}

// Two weights to an f16 pair without integer-to-float conversions: the two
// code bytes (selected by sel from x) are placed under the f16 exponent of
// 1024, where the spacing is 1, so 0x64XX reads 1024 + XX exactly; the offset
// (1024 + 128 for a q8_0 code stored XOR 0x80, 1024 + 8 for a q4_0 nibble) is
// subtracted exactly, leaving the signed code q (or q - 8); the product with
// the block scale d is then rounded once, RN(q * d): the same f16 value as
// rounding the (exact) f32 product q * d.
__device__ __forceinline__ uint32_t codes_to_h2(uint32_t x, uint32_t sel, __half2 off, __half2 d2) {
  const uint32_t h = __byte_perm(x, 0x64646464u, sel);
  const __half2 v = __hmul2_rn(__hsub2_rn(*reinterpret_cast<const __half2*>(&h), off), d2);
  return *reinterpret_cast<const uint32_t*>(&v);
}

// 8 consecutive weights of one block (8 code bytes of q8_0, or the 8 low or
// high nibbles, nsh = 0 or 4, of 8 bytes of q4_0) scaled by d -> 4 f16 pairs.
template <int BMODE>
__device__ __forceinline__ void unpack8(uint2 q, int nsh, __half2 d2, uint32_t (&w)[4]) {
  uint32_t x0, x1;
  __half2 off;
  if (BMODE == B_Q8) {
    x0 = q.x ^ 0x80808080u;
    x1 = q.y ^ 0x80808080u;
    off = __half2half2(__ushort_as_half(static_cast<unsigned short>(0x6480)));  // 1152
  } else {
    x0 = (q.x >> nsh) & 0x0F0F0F0Fu;
    x1 = (q.y >> nsh) & 0x0F0F0F0Fu;
    off = __half2half2(__ushort_as_half(static_cast<unsigned short>(0x6408)));  // 1032
  }
  w[0] = codes_to_h2(x0, 0x4140u, off, d2);
  w[1] = codes_to_h2(x0, 0x4342u, off, d2);
  w[2] = codes_to_h2(x1, 0x4140u, off, d2);
  w[3] = codes_to_h2(x1, 0x4342u, off, d2);
}

// The same 8 weights rounded once to bf16: each code is made an exact f32
// (the byte under the exponent of 2^23, where the spacing is 1, minus the
// offset), multiplied by the scale (exact: an 8-bit integer times an 11-bit
// significand) and rounded to bf16, RN(q * d).
template <int BMODE>
__device__ __forceinline__ void unpack8_bf16(uint2 q, int nsh, float d, uint32_t (&w)[4]) {
  uint32_t x[2];
  float off;
  if (BMODE == B_Q8) {
    x[0] = q.x ^ 0x80808080u;
    x[1] = q.y ^ 0x80808080u;
    off = 8388608.0f + 128.0f;
  } else {
    x[0] = (q.x >> nsh) & 0x0F0F0F0Fu;
    x[1] = (q.y >> nsh) & 0x0F0F0F0Fu;
    off = 8388608.0f + 8.0f;
  }
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    float v[4];
#pragma unroll
    for (int b = 0; b < 4; ++b) v[b] = (__uint_as_float(__byte_perm(x[h], 0x4B000000u, 0x7540u + b)) - off) * d;
    w[2 * h] = pack2<true>(v[0], v[1]);
    w[2 * h + 1] = pack2<true>(v[2], v[3]);
  }
}

// Address of the 8 codes of weights k..k+7 (k % 8 == 0) of row n, and the
// nibble shift for q4_0 (byte j of a block holds elements j and j + 16).
template <int BMODE>
__device__ __forceinline__ const uint2* quant_src(const void* bq, int K, int n, int k, int& nsh) {
  if (BMODE == B_Q8) {
    nsh = 0;
    return reinterpret_cast<const uint2*>(static_cast<const int8_t*>(bq) + static_cast<size_t>(n) * K + k);
  }
  const int j0 = k & 31;
  nsh = j0 >= 16 ? 4 : 0;
  return reinterpret_cast<const uint2*>(static_cast<const uint8_t*>(bq) + static_cast<size_t>(n) * (K >> 1) +
                                        (k >> 5) * 16 + (j0 & 15));
}

// Unpack a [rows x 64] slice (rows n0 .. n0 + rows - 1, K block kb) of a q8_0
// / q4_0 weight matrix into the swizzled f16 B tile.  Each thread converts 8
// consecutive K elements of one row per step: value = q * d (q8_0) or
// (q - 8) * d (q4_0), rounded once to f16.
template <int BMODE, int ROWS, bool BF>
__device__ __forceinline__ void fill_b_quant(uint8_t* sB, const GemmParams& p, int n0, int kb, int ct) {
  const int K = p.K;
  const uint32_t sbase = smem_u32(sB);
#pragma unroll 4
  for (int idx = ct; idx < ROWS * 8; idx += 128) {
    const int r = idx >> 3, u = idx & 7;
    const int n = n0 + r;
    const int k = kb * 64 + u * 8;
    const __half d = p.bscale[static_cast<size_t>(n) * (K >> 5) + (k >> 5)];
    int nsh;
    const uint2 q = __ldg(quant_src<BMODE>(p.bq, K, n, k, nsh));
    uint32_t w[4];
    if constexpr (BF)
      unpack8_bf16<BMODE>(q, nsh, __half2float(d), w);
    else
      unpack8<BMODE>(q, nsh, __half2half2(d), w);
    st_shared_v4(sbase + sw128_offset(r, u * 8), w[0], w[1], w[2], w[3]);
  }
}

// Epilogue of one output tile for one thread: its row, half of the BN
// columns (chalf), read from TMEM at tb (lane quadrant already applied).
template <int BN, bool LOWREG, bool ROPE, bool BF>
__device__ __forceinline__ void epilogue_tile(const GemmParams& p, uint32_t tb, int row, int nb, int chalf) {
  if (p.epi == EPI_RESID_F32) {
    // residual add: the residual's loads are issued before the TMEM load
    // so the two latencies overlap
#pragma unroll 1
    for (int c = chalf * (BN / 64); c < (chalf + 1) * (BN / 64); ++c) {
      const int col0 = nb * BN + c * 32;
      float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.out) + static_cast<size_t>(row) * p.ldo + col0);
      float4 x[8];
      if (row < p.M) {
#pragma unroll
        for (int j = 0; j < 8; ++j) x[j] = dst[j];
      }
      uint32_t r[32];
      tmem_ld32(tb + static_cast<uint32_t>(c * 32), r);
      if (row < p.M) {
        const float4* b4 = reinterpret_cast<const float4*>(p.bias + col0);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float4 b = p.bias ? __ldg(b4 + j) : make_float4(0.f, 0.f, 0.f, 0.f);
          x[j].x += __uint_as_float(r[4 * j]) + b.x;
          x[j].y += __uint_as_float(r[4 * j + 1]) + b.y;
          x[j].z += __uint_as_float(r[4 * j + 2]) + b.z;
          x[j].w += __uint_as_float(r[4 * j + 3]) + b.w;
          dst[j] = x[j];
        }
      }
    }
  } else {
#pragma unroll 1
    for (int c = chalf * (BN / 64); c < (chalf + 1) * (BN / 64); ++c) {
      uint32_t r[32];
      tmem_ld32(tb + static_cast<uint32_t>(c * 32), r);
      if (row < p.M) epilogue_chunk<LOWREG, ROPE, BF>(p, row, nb * BN + c * 32, r);
    }
  }
}

// Bias of 32 consecutive output columns (zeros without a bias).
__device__ __forceinline__ void load_bias32(const float* bias, int col0, float4 (&bb)[8]) {
#pragma unroll
  for (int j = 0; j < 8; ++j)
    bb[j] = bias ? __ldg(reinterpret_cast<const float4*>(bias + col0) + j) : make_float4(0.f, 0.f, 0.f, 0.f);
}

// TMA epilogue of one output tile for one warp: 32 rows starting at row0,
// half of the BN columns (chalf).  Each 32-row x 128-byte chunk (32 f32
// columns, or 64 f16 columns) is written to the warp's staging buffer in the
// 128-byte-swizzled layout and sent with one TMA store (f16 / f32 outputs)
// or one TMA reduce-add (f32 residual: X += A W^T + b), so every global
// write is a full, coalesced line.
template <int BN, bool LOWREG, bool BF>
__device__ __forceinline__ void epilogue_tile_tma(const GemmParams& p, const CUtensorMap* tmC, uint32_t tb,
                                                  int row0, int nb, int chalf, uint8_t* stage_buf, int lane,
                                                  bool& pending) {
  const uint32_t sb = smem_u32(stage_buf);
  const uint32_t row_off = static_cast<uint32_t>(lane) * 128u;
  const bool live = row0 < p.M;
  const int c_begin = chalf * (BN / 64), c_end = (chalf + 1) * (BN / 64);
  if (p.epi == EPI_F32 || p.epi == EPI_RESID_F32) {
#pragma unroll 1
    for (int c = c_begin; c < c_end; ++c) {
      const int col0 = nb * BN + c * 32;
      // the bias loads are issued first so that their latency overlaps the
      // TMEM load's (after it in the 128-register kernels)
      float4 bb[8];
      if (!LOWREG) load_bias32(p.bias, col0, bb);
      uint32_t r[32];
      tmem_ld32(tb + static_cast<uint32_t>(c * 32), r);
      float v[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
      if (!LOWREG || p.bias) {
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float4 b = LOWREG ? __ldg(reinterpret_cast<const float4*>(p.bias + col0) + j) : bb[j];
          v[4 * j] += b.x;
          v[4 * j + 1] += b.y;
          v[4 * j + 2] += b.z;
          v[4 * j + 3] += b.w;
        }
      }
      if (pending) {  // the previous chunk's store must have read the buffer
        if (lane == 0) bulk_wait_read0();
        __syncwarp();
      }
#pragma unroll
      for (int u = 0; u < 8; ++u)
        st_shared_v4(sb + row_off + static_cast<uint32_t>(((u ^ (lane & 7)) & 7) << 4), __float_as_uint(v[4 * u]),
                     __float_as_uint(v[4 * u + 1]), __float_as_uint(v[4 * u + 2]), __float_as_uint(v[4 * u + 3]));
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0 && live) {
        if (p.epi == EPI_RESID_F32)
          tma_reduce_add_2d(tmC, stage_buf, col0, row0);
        else
          tma_store_2d(tmC, stage_buf, col0, row0);
        bulk_commit();
      }
      pending = true;
    }
  } else {  // f16 output: two 32-column TMEM chunks per 128-byte staging row
#pragma unroll 1
    for (int c = c_begin; c < c_end; c += 2) {
      uint32_t w[32];
      const int col0 = nb * BN + c * 32;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        float4 bb[8];  // issued before the TMEM load so the two latencies overlap
        if (!LOWREG) load_bias32(p.bias, col0 + h * 32, bb);
        uint32_t r[32];
        tmem_ld32(tb + static_cast<uint32_t>((c + h) * 32), r);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          uint64_t lo = f2_pack(__uint_as_float(r[4 * j]), __uint_as_float(r[4 * j + 1]));
          uint64_t hi = f2_pack(__uint_as_float(r[4 * j + 2]), __uint_as_float(r[4 * j + 3]));
          if (!LOWREG) {
            lo = f2_add(lo, f2_pack(bb[j].x, bb[j].y));
            hi = f2_add(hi, f2_pack(bb[j].z, bb[j].w));
          } else if (p.bias) {
            const float4 b = __ldg(reinterpret_cast<const float4*>(p.bias + col0 + h * 32) + j);
            lo = f2_add(lo, f2_pack(b.x, b.y));
            hi = f2_add(hi, f2_pack(b.z, b.w));
          }
          float x0, x1, x2, x3;
          f2_unpack(lo, x0, x1);
          f2_unpack(hi, x2, x3);
          if (p.epi == EPI_GELU_F16) {
            gelu_pair<LOWREG>(x0, x1);
            gelu_pair<LOWREG>(x2, x3);
          }
          w[h * 16 + 2 * j] = pack2<BF>(x0, x1);
          w[h * 16 + 2 * j + 1] = pack2<BF>(x2, x3);
        }
      }
      if (pending) {
        if (lane == 0) bulk_wait_read0();
        __syncwarp();
      }
#pragma unroll
      for (int u = 0; u < 8; ++u)
        st_shared_v4(sb + row_off + static_cast<uint32_t>(((u ^ (lane & 7)) & 7) << 4), w[4 * u], w[4 * u + 1],
                     w[4 * u + 2], w[4 * u + 3]);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0 && live) {
        tma_store_2d(tmC, stage_buf, col0, row0);
        bulk_commit();
      }
      pending = true;
    }
  }
}

// QKV epilogue of one output tile for one warp (32 rows from row0, half of
// the BN columns).  Per head and 32 token rows, Q and K are one 32 x 128-byte
// tile of [B*h, N, 64]: staged like the f16 epilogue and sent with one 3-D
// TMA store at (0, t0, b*h + head) when the 32 rows lie in one clip, else
// written row by row.  V goes to V^T [B*h, 64, Npad] column by column (one
// coalesced 64-byte store per dimension and warp).
template <int BN, bool LOWREG, bool ROPE, bool BF>
__device__ __forceinline__ void epilogue_tile_qkv(const GemmParams& p, const CUtensorMap* tmQ, const CUtensorMap* tmK,
                                                  uint32_t tb, int row0, int nb, int chalf, uint8_t* stage_buf,
                                                  int lane, bool& pending) {
  const uint32_t sb = smem_u32(stage_buf);
  const uint32_t row_off = static_cast<uint32_t>(lane) * 128u;
  const int ntok = p.qkv.ntok, heads = p.qkv.heads;
  const int row = row0 + lane;
  const int b0 = row0 / ntok, t0 = row0 - b0 * ntok;
  const bool one_clip = row0 + 31 < p.M && t0 + 31 < ntok;
  const int c_begin = chalf * (BN / 64), c_end = (chalf + 1) * (BN / 64);
#pragma unroll 1
  for (int c = c_begin; c < c_end; c += 2) {
    const int col0 = nb * BN + c * 32;
    const int part = col0 / p.qkv.dim + p.qkv.first_part;
    const int within = col0 % p.qkv.dim;
    const int hd = within >> 6;
    if (part == 2) {
#pragma unroll 1
      for (int h = 0; h < 2; ++h) {
        float4 bb[8];
        if (!LOWREG) load_bias32(p.bias, col0 + h * 32, bb);
        uint32_t r[32];
        tmem_ld32(tb + static_cast<uint32_t>((c + h) * 32), r);
        if (LOWREG) load_bias32(p.bias, col0 + h * 32, bb);
        if (row < p.M && p.qkv.vt) {
          const int b = row / ntok, t = row - b * ntok;
          __half* base = p.qkv.vt + ((static_cast<size_t>(b) * heads + hd) * 64 + h * 32) * p.qkv.npad + t;
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            base[static_cast<size_t>(4 * j) * p.qkv.npad] = __ushort_as_half(pack1<BF>(__uint_as_float(r[4 * j]) + bb[j].x));
            base[static_cast<size_t>(4 * j + 1) * p.qkv.npad] = __ushort_as_half(pack1<BF>(__uint_as_float(r[4 * j + 1]) + bb[j].y));
            base[static_cast<size_t>(4 * j + 2) * p.qkv.npad] = __ushort_as_half(pack1<BF>(__uint_as_float(r[4 * j + 2]) + bb[j].z));
            base[static_cast<size_t>(4 * j + 3) * p.qkv.npad] = __ushort_as_half(pack1<BF>(__uint_as_float(r[4 * j + 3]) + bb[j].w));
          }
        }
      }
      continue;
    }
    __half* base = part == 0 ? p.qkv.q : p.qkv.k;
    int pt = 0, py = 0, px = 0;
    if (ROPE) rope_position(p.qkv, min(row, p.M - 1), pt, py, px);
    uint32_t w[32];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      float4 bb[8];
      if (!LOWREG) load_bias32(p.bias, col0 + h * 32, bb);
      uint32_t r[32];
      tmem_ld32(tb + static_cast<uint32_t>((c + h) * 32), r);
      if (LOWREG) load_bias32(p.bias, col0 + h * 32, bb);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        float x0 = __uint_as_float(r[4 * j]) + bb[j].x, x1 = __uint_as_float(r[4 * j + 1]) + bb[j].y;
        float x2 = __uint_as_float(r[4 * j + 2]) + bb[j].z, x3 = __uint_as_float(r[4 * j + 3]) + bb[j].w;
        if (ROPE) {  // q and k of a rotary model
          rope_pair(x0, x1, h * 32 + 4 * j, pt, py, px, p.qkv.rope);
          rope_pair(x2, x3, h * 32 + 4 * j + 2, pt, py, px, p.qkv.rope);
        }
        w[h * 16 + 2 * j] = pack2<BF>(x0, x1);
        w[h * 16 + 2 * j + 1] = pack2<BF>(x2, x3);
      }
    }
    if (!base) continue;
    if (one_clip) {  // warp-uniform
      if (pending) {
        if (lane == 0) bulk_wait_read0();
        __syncwarp();
      }
#pragma unroll
      for (int u = 0; u < 8; ++u)
        st_shared_v4(sb + row_off + static_cast<uint32_t>(((u ^ (lane & 7)) & 7) << 4), w[4 * u], w[4 * u + 1],
                     w[4 * u + 2], w[4 * u + 3]);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        tma_store_3d(part == 0 ? tmQ : tmK, stage_buf, 0, t0, b0 * heads + hd);
        bulk_commit();
      }
      pending = true;
    } else if (row < p.M) {
      const int b = row / ntok, t = row - b * ntok;
      uint4* dst = reinterpret_cast<uint4*>(base + ((static_cast<size_t>(b) * heads + hd) * ntok + t) * 64);
#pragma unroll
      for (int u = 0; u < 8; ++u) dst[u] = make_uint4(w[4 * u], w[4 * u + 1], w[4 * u + 2], w[4 * u + 3]);
    }
  }
}

template <int BN, int BMODE, bool ROPE, bool BF>
__global__ void __launch_bounds__(BMODE != B_F16 ? 448 : 320, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const __grid_constant__ CUtensorMap tmC, const __grid_constant__ CUtensorMap tmC2,
                   const GemmParams p) {
  using C = GemmCfg<BN>;
  constexpr bool CONV = BMODE != B_F16;
  constexpr int S = C::STAGES;
  extern __shared__ uint8_t dsmem[];
  __shared__ uint64_t full_bar[S], conv_bar[S], empty_bar[S], tfull_bar[2], tempty_bar[2], drain_bar;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;

  const uint32_t raw = smem_u32(dsmem);
  uint8_t* smem = dsmem + ((1024u - (raw & 1023u)) & 1023u);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&conv_bar[s], 128);
      mbar_init(&empty_bar[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull_bar[a], 1);
      mbar_init(&tempty_bar[a], 256);
    }
    mbar_init(&drain_bar, 1);
    abort_sh = 0;
    mbar_fence_init();
  }
  if (warp == 1) {
    tmem_alloc(&tmem_base_sh, C::TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    if (BMODE == B_F16) tma_prefetch_desc(&tmB);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = tmem_base_sh;
  pdl_wait();  // A (and a residual output) come from the previous kernel
  pdl_trigger();

  WaitCtl w;
  w.abort = reinterpret_cast<volatile int*>(&abort_sh);
  w.err = p.err;
  w.timeout_ns = p.timeout_ns;
  w.where = (KID_GEMM << 8) | static_cast<unsigned>(warp);
  const int num_tiles = p.m_tiles * p.n_tiles;
  const int kblocks = p.K / 64;

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0, armed = 0, armed_par = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
        const int nb = t % p.n_tiles, mb = t / p.n_tiles;
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait(&empty_bar[stage], phase ^ 1, w)) {
            ok = false;
            break;
          }
          uint8_t* sA = smem + stage * C::STAGE_BYTES;
          uint8_t* sB = sA + C::A_BYTES;
          constexpr uint32_t tx = (uint32_t)C::A_BYTES + (BMODE == B_F16 ? (uint32_t)C::B_BYTES : 0u);
          mbar_expect_tx(&full_bar[stage], tx);
          tma_load_2d(sA, &tmA, &full_bar[stage], kb * 64, mb * 128);
          if (BMODE == B_F16) tma_load_2d(sB, &tmB, &full_bar[stage], kb * 64, nb * BN);
          armed |= 1u << stage;
          armed_par = (armed_par & ~(1u << stage)) | (phase << stage);
          if (++stage == S) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      if (!ok) {  // let the copies already issued land before the CTA exits
        for (int s = 0; s < S; ++s)
          if ((armed >> s) & 1u) mbar_wait_drain(&full_bar[s], (armed_par >> s) & 1u);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_f16_f32(128, BN, BF);
      int stage = 0, acc = 0;
      uint32_t phase = 0, aphase = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
        if (!mbar_wait(&tempty_bar[acc], aphase ^ 1, w)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t dtm = tmem_base + static_cast<uint32_t>(acc * BN);
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait(&full_bar[stage], phase, w)) {
            ok = false;
            break;
          }
          if (CONV && !mbar_wait(&conv_bar[stage], phase, w)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(smem + stage * C::STAGE_BYTES);
          const uint64_t ad = sdesc_kmajor_sw128(a0);
          const uint64_t bd = sdesc_kmajor_sw128(a0 + C::A_BYTES);
#pragma unroll
          for (int k = 0; k < 4; ++k)
            tc_mma_f16_ss(dtm, ad + static_cast<uint64_t>(2 * k), bd + static_cast<uint64_t>(2 * k), idesc,
                          (kb | k) != 0 ? 1u : 0u);
          tc_commit(&empty_bar[stage]);
          if (++stage == S) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        tc_commit(&tfull_bar[acc]);
        if (++acc == 2) {
          acc = 0;
          aphase ^= 1;
        }
      }
      // every MMA issued above completes before TMEM is released
      tc_commit(&drain_bar);
      mbar_wait_drain(&drain_bar, 0);
    }
  } else if (warp < 10) {
    // 8 epilogue warps: warps w and w+4 read the same TMEM lane quadrant
    // (w % 4) and split the tile's columns in two halves.
    const int quad = warp & 3;
    const int chalf = (warp - 2) >> 2;
    uint8_t* stage_buf = smem + S * C::STAGE_BYTES + (warp - 2) * 4096;
    bool pending = false;
    int acc = 0;
    uint32_t aphase = 0;
    for (int t = blockIdx.x; t < num_tiles; t += gridDim.x) {
      bool ok = mbar_wait(&tfull_bar[acc], aphase, w);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      const int nb = t % p.n_tiles, mb = t / p.n_tiles;
      const int row = mb * 128 + quad * 32 + lane;
      const uint32_t tb = tmem_base + static_cast<uint32_t>(acc * BN) + (static_cast<uint32_t>(quad * 32) << 16);
      constexpr bool kLowReg = BMODE != B_F16;
      bool done = false;
      if constexpr (!kLowReg) {  // the 128-register kernels keep the row-by-row QKV stores
        if (p.tma_epi && p.epi == EPI_QKV) {
          epilogue_tile_qkv<BN, false, ROPE, BF>(p, &tmC, &tmC2, tb, mb * 128 + quad * 32, nb, chalf, stage_buf, lane,
                                             pending);
          done = true;
        }
      }
      if (done) {
      } else if (p.tma_epi && p.epi != EPI_QKV)
        epilogue_tile_tma<BN, kLowReg, BF>(p, &tmC, tb, mb * 128 + quad * 32, nb, chalf, stage_buf, lane, pending);
      else
        epilogue_tile<BN, kLowReg, ROPE, BF>(p, tb, row, nb, chalf);
      tc_fence_before();
      mbar_arrive(&tempty_bar[acc]);
      if (++acc == 2) {
        acc = 0;
        aphase ^= 1;
      }
    }
    if (pending && lane == 0) bulk_wait0();
  } else if (CONV) {
    const int ct = threadIdx.x - 320;
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
      const int nb = t % p.n_tiles;
      for (int kb = 0; kb < kblocks; ++kb) {
        bool okw = mbar_wait(&empty_bar[stage], phase ^ 1, w);
        okw = __all_sync(0xffffffffu, okw);
        if (!okw) {
          ok = false;
          break;
        }
        uint8_t* sB = smem + stage * C::STAGE_BYTES + C::A_BYTES;
        fill_b_quant<BMODE, BN, BF>(sB, p, nb * BN, kb, ct);
        fence_proxy_async_smem();
        mbar_arrive(&conv_bar[stage]);
        if (++stage == S) {
          stage = 0;
          phase ^= 1;
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}


// ---------------------------------------------------------------------------
// CTA-pair variant: a cluster of two CTAs on two SMs computes a 256 x BN
// tile with tcgen05.mma.cta_group::2 (M = 256).  Each CTA holds the 128 A
// rows of its half and half of the B tile (BN/2 rows), so per SM a stage is
// 16 KB + BN*64 bytes instead of 16 KB + BN*128: the same MMA work per SM
// with two thirds of the shared-memory traffic and more stages in flight.
// The leader CTA (rank 0) issues the MMAs; its commits arrive on the
// barriers of both CTAs (multicast commit).  TMA loads are plain (no
// multicast): each CTA loads its own tiles, the bytes counted on the
// leader's barrier.
//
// B operand: f16 weights come by TMA (BMODE B_F16, 320 threads).  q8_0 /
// q4_0 weights (BMODE B_Q8 / B_Q4, 448 threads) are unpacked in the loader:
// a second producer lane stages the codes and scale groups of the CTA's
// BN/2 weight rows by TMA into a ring of their own, four converter warps
// per CTA unpack them (shared memory to shared memory) into the swizzled
// f16 B tile of the MMA ring, and each converter warp then arrives on the
// leader's conversion barrier (cluster scope), which the MMA issuer waits
// for beside the TMA barrier of the A tiles.
template <int BN, int BMODE>
struct Gemm2Cfg {
  static constexpr bool CONV = BMODE != B_F16;
  static constexpr int A_BYTES = 128 * 64 * 2;
  static constexpr int B_BYTES = (BN / 2) * 64 * 2;
  // quantised weights: the raw codes of this CTA's BN/2 rows for one K block
  // (64 bytes a row for q8_0, 32 for q4_0) and a 16-byte group of 8 scales
  // a row holding the K block's two scales, both staged by TMA
  static constexpr int RAW_W = BMODE == B_Q8 ? 64 : 32;
  static constexpr int RAW_BYTES = CONV ? (BN / 2) * RAW_W : 0;
  static constexpr int SC_BYTES = CONV ? (BN / 2) * 16 : 0;
  // a stage of the MMA ring: the A tile and this CTA's half of the B tile
  static constexpr int STAGE_BYTES = (A_BYTES + B_BYTES + 1023) / 1024 * 1024;
  static constexpr int STAGING = 8 * 4096;  // epilogue staging
  // quantised: four or five MMA stages, converter warp w filling the B tiles
  // of K blocks w, w + 4, ...; the codes and scales come through a ring of
  // their own, as deep as the rest of shared memory allows, freed by the
  // converter warps as soon as a K block is unpacked, so their loads run
  // ahead of the MMA ring (q4_0's smaller code tiles leave room for a fifth
  // MMA stage beside five code stages; q8_0 keeps four MMA stages and six
  // code stages).
  static constexpr int STAGES = CONV ? (BMODE == B_Q4 ? 5 : 4) : (BN == 256 ? 6 : (BN == 192 ? 6 : 8));
  static constexpr int RAW_STAGE_BYTES = CONV ? (RAW_BYTES + SC_BYTES + 1023) / 1024 * 1024 : 0;
  static constexpr int RSTAGES_FIT =
      CONV ? (227 * 1024 - STAGES * STAGE_BYTES - STAGING - 1024) / (RAW_STAGE_BYTES > 0 ? RAW_STAGE_BYTES : 1) : 0;
  static constexpr int RSTAGES = CONV ? (RSTAGES_FIT > 8 ? 8 : RSTAGES_FIT) : 0;
  // At least as many code slots as converter warps: the converter warp of K
  // block i last waited for block i - 4, so with RSTAGES >= 4 the previous fill
  // of slot i % RSTAGES (block i - RSTAGES) has landed and the slot's barrier is
  // never two phases behind the parity the warp waits for.  A shallower ring
  // lets a warp see an old phase as complete.
  static_assert(!CONV || RSTAGES >= 4, "the code ring needs at least as many slots as converter warps");
  static constexpr int TMEM_COLS = 2 * BN <= 256 ? 256 : 512;
  static constexpr int SMEM = STAGES * STAGE_BYTES + RSTAGES * RAW_STAGE_BYTES + STAGING + 1024;
  static constexpr int THREADS = CONV ? 448 : 320;
};

// One converter warp unpacks a whole stage: this CTA's BN/2 weight rows of
// one K block, read from the staged codes and scales, to f16 in the
// swizzled B tile.  Lane l takes the K offset 8 (l % 8) of rows l / 8 + 4 j.
// The rows go in batches of eight whose shared-memory loads are all issued
// before the batch is converted, the next batch's loads before this batch's
// stores: the loads and stores are ordered asm statements, so without the
// batching each row's load would wait for the previous row's store and the
// unpack of a stage would run at shared-memory latency.
template <int BMODE, int ROWS, bool BF>
__device__ __forceinline__ void quant_stage_convert(const uint8_t* sRaw, const uint8_t* sSc, uint8_t* sB, int kb,
                                                    int lane) {
  constexpr int RAW_W = BMODE == B_Q8 ? 64 : 32;
  constexpr int kBatch = 8, kBatches = ROWS / (4 * kBatch);
  static_assert(ROWS % (4 * kBatch) == 0, "rows of a stage in whole batches");
  const uint32_t raw = smem_u32(sRaw), sc = smem_u32(sSc), sbase = smem_u32(sB);
  const int u = lane & 7, r0 = lane >> 3;
  // q8_0: bytes 8u..8u+7 of the row's 64; q4_0: the K offset's block (u / 4)
  // holds 16 bytes, its elements j and j + 16 in byte j (low, high nibble)
  const int off = BMODE == B_Q8 ? 8 * u : 16 * (u >> 2) + 8 * (u & 1);
  const int nsh = (BMODE == B_Q4 && (u & 2)) ? 4 : 0;
  const int sidx = ((2 * kb) & 7) + (u >> 2);  // the unit's scale in the row's group of 8
  uint2 q[2][kBatch];
  unsigned short dbits[2][kBatch];
  auto load = [&](int b, uint2 (&qb)[kBatch], unsigned short (&db)[kBatch]) {
#pragma unroll
    for (int j = 0; j < kBatch; ++j) {
      const int r = r0 + 4 * (kBatch * b + j);
      asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(qb[j].x), "=r"(qb[j].y) : "r"(raw + r * RAW_W + off));
      asm volatile("ld.shared.u16 %0, [%1];" : "=h"(db[j]) : "r"(sc + r * 16 + sidx * 2));
    }
  };
  load(0, q[0], dbits[0]);
#pragma unroll
  for (int b = 0; b < kBatches; ++b) {
    if (b + 1 < kBatches) load(b + 1, q[(b + 1) & 1], dbits[(b + 1) & 1]);
#pragma unroll
    for (int j = 0; j < kBatch; ++j) {
      const int r = r0 + 4 * (kBatch * b + j);
      uint32_t w[4];
      if constexpr (BF)
        unpack8_bf16<BMODE>(q[b & 1][j], nsh, __half2float(__ushort_as_half(dbits[b & 1][j])), w);
      else
        unpack8<BMODE>(q[b & 1][j], nsh, __half2half2(__ushort_as_half(dbits[b & 1][j])), w);
      st_shared_v4(sbase + sw128_offset(r, u * 8), w[0], w[1], w[2], w[3]);
    }
  }
}

// Wait on a local barrier whose arrivals come from another CTA of the
// cluster (acquire at cluster scope); bounded like mbar_wait.
__device__ __forceinline__ bool mbar_try_wait_cluster(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ bool mbar_wait_cluster(uint64_t* bar, uint32_t parity, const WaitCtl& w) {
  if (w.timeout_ns == 0) {
    if (mbar_try_wait_cluster(bar, parity)) return true;
    raise_error(w, DERR_TIMEOUT);
    return false;
  }
  const unsigned long long t0 = globaltimer();
  while (true) {
    if (mbar_try_wait_cluster(bar, parity)) return true;
    if (*w.abort) return false;
    if (globaltimer() - t0 > w.timeout_ns) {
      raise_error(w, DERR_TIMEOUT);
      return false;
    }
  }
}

template <int BN, bool ROPE, int BMODE, bool BF>
__global__ void __launch_bounds__(Gemm2Cfg<BN, BMODE>::THREADS, 1)
    gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                     const __grid_constant__ CUtensorMap tmC, const __grid_constant__ CUtensorMap tmC2,
                     const __grid_constant__ CUtensorMap tmS, const GemmParams p) {
  using C = Gemm2Cfg<BN, BMODE>;
  constexpr int S = C::STAGES;
  constexpr bool CONV = C::CONV;
  extern __shared__ uint8_t dsmem[];
  constexpr int RS = C::RSTAGES > 0 ? C::RSTAGES : 1;
  __shared__ uint64_t full_bar[S], empty_bar[S], conv_bar[S], raw_full[RS], raw_empty[RS], tfull_bar[2], tempty_bar[2],
      drain_bar;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;

  const uint32_t raw = smem_u32(dsmem);
  uint8_t* smem = dsmem + ((1024u - (raw & 1023u)) & 1023u);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();  // 0: leader (issues the MMAs), 1: peer

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full_bar[s], 1);     // leader: one expect-tx arrival + the bytes of both CTAs
      mbar_init(&empty_bar[s], 1);    // both: the leader's multicast commit
      mbar_init(&conv_bar[s], 2);     // leader: the stage's converter warp in each CTA
    }
    for (int r = 0; r < RS; ++r) {
      mbar_init(&raw_full[r], 1);     // both: this CTA's codes and scales (expect-tx + bytes)
      mbar_init(&raw_empty[r], 1);    // both: the converter warp that unpacked the slot
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull_bar[a], 1);    // both: the leader's multicast commit
      mbar_init(&tempty_bar[a], 16);  // leader: one arrival per epilogue warp of both CTAs
    }
    mbar_init(&drain_bar, 1);
    abort_sh = 0;
    mbar_fence_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(&tmem_base_sh, C::TMEM_COLS);
    tmem_relinquish_pair();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    if (CONV) tma_prefetch_desc(&tmS);
  }
  tc_fence_before();
  cluster_sync();  // barriers of both CTAs initialised before any remote arrival
  tc_fence_after();
  const uint32_t tmem_base = tmem_base_sh;
  pdl_wait();  // A (and a residual output) come from the previous kernel
  pdl_trigger();

  WaitCtl w;
  w.abort = reinterpret_cast<volatile int*>(&abort_sh);
  w.err = p.err;
  w.timeout_ns = p.timeout_ns;
  w.where = (KID_GEMM << 8) | 0x80u | static_cast<unsigned>(warp);
  const int num_tiles = ((p.M + 255) / 256) * p.n_tiles;
  const int n_clusters = gridDim.x >> 1;
  const int cid = blockIdx.x >> 1;
  const int kblocks = p.K / 64;

  if (warp == 0) {
    if (lane == 0) {
      const uint32_t leader_full0 = mapa_shared(smem_u32(&full_bar[0]), 0);
      int stage = 0;
      uint32_t phase = 0, armed = 0, armed_par = 0;
      bool ok = true;
      for (int t = cid; t < num_tiles && ok; t += n_clusters) {
        const int nb = t % p.n_tiles, mb = t / p.n_tiles;
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait(&empty_bar[stage], phase ^ 1, w)) {
            ok = false;
            break;
          }
          uint8_t* sA = smem + stage * C::STAGE_BYTES;
          uint8_t* sB = sA + C::A_BYTES;
          if (rank == 0) mbar_expect_tx(&full_bar[stage], CONV ? 2u * C::A_BYTES : 2u * (C::A_BYTES + C::B_BYTES));
          const uint32_t fb = leader_full0 + static_cast<uint32_t>(stage * sizeof(uint64_t));
          tma_load_2d_pair(sA, &tmA, fb, kb * 64, mb * 256 + static_cast<int>(rank) * 128);
          if (!CONV) tma_load_2d_pair(sB, &tmB, fb, kb * 64, nb * BN + static_cast<int>(rank) * (BN / 2));
          armed |= 1u << stage;
          armed_par = (armed_par & ~(1u << stage)) | (phase << stage);
          if (++stage == S) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      if (!ok && rank == 0) {  // let the copies already counted on the barriers land
        for (int s = 0; s < S; ++s)
          if ((armed >> s) & 1u) mbar_wait_drain(&full_bar[s], (armed_par >> s) & 1u);
      }
    } else if (CONV && lane == 1) {
      // this CTA's codes and scales of every K block, through their own ring
      uint8_t* raw_ring = smem + S * C::STAGE_BYTES;
      int r = 0;
      uint32_t rphase = 0, armed = 0, armed_par = 0;
      bool ok = true;
      for (int t = cid; t < num_tiles && ok; t += n_clusters) {
        const int nb = t % p.n_tiles;
        const int n0 = nb * BN + static_cast<int>(rank) * (BN / 2);
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait(&raw_empty[r], rphase ^ 1, w)) {
            ok = false;
            break;
          }
          uint8_t* sRaw = raw_ring + r * C::RAW_STAGE_BYTES;
          mbar_expect_tx(&raw_full[r], static_cast<uint32_t>(C::RAW_BYTES + C::SC_BYTES));
          tma_load_2d(sRaw, &tmB, &raw_full[r], kb * C::RAW_W, n0);
          tma_load_2d(sRaw + C::RAW_BYTES, &tmS, &raw_full[r], (2 * kb) & ~7, n0);
          armed |= 1u << r;
          armed_par = (armed_par & ~(1u << r)) | (rphase << r);
          if (++r == RS) {
            r = 0;
            rphase ^= 1;
          }
        }
      }
      if (!ok) {
        for (int s = 0; s < RS; ++s)
          if ((armed >> s) & 1u) mbar_wait_drain(&raw_full[s], (armed_par >> s) & 1u);
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      constexpr uint32_t idesc = idesc_f16_f32(256, BN, BF);
      int stage = 0, acc = 0;
      uint32_t phase = 0, aphase = 0;
      bool ok = true;
      for (int t = cid; t < num_tiles && ok; t += n_clusters) {
        if (!mbar_wait(&tempty_bar[acc], aphase ^ 1, w)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t dtm = tmem_base + static_cast<uint32_t>(acc * BN);
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait(&full_bar[stage], phase, w)) {
            ok = false;
            break;
          }
          if (CONV && !mbar_wait_cluster(&conv_bar[stage], phase, w)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(smem + stage * C::STAGE_BYTES);
          const uint64_t ad = sdesc_kmajor_sw128(a0);
          const uint64_t bd = sdesc_kmajor_sw128(a0 + C::A_BYTES);
#pragma unroll
          for (int k = 0; k < 4; ++k)
            tc_mma_f16_ss_pair(dtm, ad + static_cast<uint64_t>(2 * k), bd + static_cast<uint64_t>(2 * k), idesc,
                               (kb | k) != 0 ? 1u : 0u);
          tc_commit_pair_mc(&empty_bar[stage], 0x3);
          if (++stage == S) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        tc_commit_pair_mc(&tfull_bar[acc], 0x3);
        if (++acc == 2) {
          acc = 0;
          aphase ^= 1;
        }
      }
      tc_commit_pair_mc(&drain_bar, 0x1);
      mbar_wait_drain(&drain_bar, 0);
    }
  } else if (warp < 10) {
    const int quad = warp & 3;
    const int chalf = (warp - 2) >> 2;
    const uint32_t leader_tempty0 = mapa_shared(smem_u32(&tempty_bar[0]), 0);
    uint8_t* stage_buf = smem + S * C::STAGE_BYTES + C::RSTAGES * C::RAW_STAGE_BYTES + (warp - 2) * 4096;
    bool pending = false;
    int acc = 0;
    uint32_t aphase = 0;
    for (int t = cid; t < num_tiles; t += n_clusters) {
      bool ok = mbar_wait(&tfull_bar[acc], aphase, w);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      const int nb = t % p.n_tiles, mb = t / p.n_tiles;
      const int row0 = mb * 256 + static_cast<int>(rank) * 128 + quad * 32;
      const uint32_t tb = tmem_base + static_cast<uint32_t>(acc * BN) + (static_cast<uint32_t>(quad * 32) << 16);
      if (p.tma_epi && p.epi == EPI_QKV)
        epilogue_tile_qkv<BN, true, ROPE, BF>(p, &tmC, &tmC2, tb, row0, nb, chalf, stage_buf, lane, pending);
      else if (p.tma_epi)
        epilogue_tile_tma<BN, CONV, BF>(p, &tmC, tb, row0, nb, chalf, stage_buf, lane, pending);
      else
        epilogue_tile<BN, CONV, ROPE, BF>(p, tb, row0 + lane, nb, chalf);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(leader_tempty0 + static_cast<uint32_t>(acc * sizeof(uint64_t)));
      if (++acc == 2) {
        acc = 0;
        aphase ^= 1;
      }
    }
    if (pending && lane == 0) bulk_wait0();
  } else if (CONV) {
    // converter warps 10-13: warp cw takes K-block positions cw, cw + 4, ...
    // of the MMA's sequence (all in stage cw of the four), so four stages
    // convert at once; once a stage's
    // codes and scales have landed it unpacks this CTA's BN/2 weight rows
    // into the stage's f16 B tile (shared memory to shared memory) and
    // signals the leader
    const int cw = warp - 10;
    const uint32_t leader_conv0 = mapa_shared(smem_u32(&conv_bar[0]), 0);
    const int total = ((num_tiles - cid + n_clusters - 1) / n_clusters) * kblocks;  // K blocks this pair runs
    uint8_t* raw_ring = smem + S * C::STAGE_BYTES;
    for (int i = cw; i < total; i += 4) {
      const int stage = i % S, r = i % RS;
      const uint32_t phase = static_cast<uint32_t>(i / S) & 1u;
      const uint32_t rphase = static_cast<uint32_t>(i / RS) & 1u;
      // the codes have landed, and the MMA that read this stage's B tile before is done
      bool okw = mbar_wait(&raw_full[r], rphase, w) && mbar_wait(&empty_bar[stage], phase ^ 1, w);
      if (!__all_sync(0xffffffffu, okw)) break;
      uint8_t* sB = smem + stage * C::STAGE_BYTES + C::A_BYTES;
      uint8_t* sRaw = raw_ring + r * C::RAW_STAGE_BYTES;
      quant_stage_convert<BMODE, BN / 2, BF>(sRaw, sRaw + C::RAW_BYTES, sB, i % kblocks, lane);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&raw_empty[r]);
        mbar_arrive_cluster(leader_conv0 + static_cast<uint32_t>(stage * sizeof(uint64_t)));
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // neither CTA leaves while the pair's MMAs or arrivals may touch it
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, C::TMEM_COLS);
  }
}

// ------------------------------------------------------------------ host --
static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  // resolved once (a function-local static is initialised by one thread)
  static const PFN_cuTensorMapEncodeTiled_v12000 fn = []() -> PFN_cuTensorMapEncodeTiled_v12000 {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
    return nullptr;
  }();
  return fn;
}

bool make_tmap_f16(CUtensorMap* m, const void* base, int rank, const uint64_t* dims, const uint64_t* strides_bytes,
                   const uint32_t* box) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t d[3], s[2];
  cuuint32_t b[3], es[3] = {1, 1, 1};
  for (int i = 0; i < rank; ++i) {
    d[i] = dims[i];
    b[i] = box[i];
  }
  for (int i = 0; i + 1 < rank; ++i) s[i] = strides_bytes[i];
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, rank, const_cast<void*>(base), d, s, b, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool make_tmap_2d(CUtensorMap* m, const void* base, int esize, uint64_t cols, uint64_t rows, uint64_t row_bytes,
                  uint32_t box_cols, uint32_t box_rows) {
  auto fn = encode_fn();
  if (!fn || (esize != 2 && esize != 4)) return false;
  cuuint64_t d[2] = {cols, rows}, st[1] = {row_bytes};
  cuuint32_t b[2] = {box_cols, box_rows}, es[2] = {1, 1};
  CUresult r = fn(m, esize == 2 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2,
                  const_cast<void*>(base), d, st, b, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// 2-D map without swizzle (staged raw bytes: uint8 codes, f16 scale groups).
static bool make_tmap_plain(CUtensorMap* m, const void* base, CUtensorMapDataType dt, uint64_t cols, uint64_t rows,
                            uint64_t row_bytes, uint32_t box_cols, uint32_t box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t d[2] = {cols, rows}, st[1] = {row_bytes};
  cuuint32_t b[2] = {box_cols, box_rows}, es[2] = {1, 1};
  CUresult r = fn(m, dt, 2, const_cast<void*>(base), d, st, b, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

int num_sms() {
  int dev = 0, n = 0;
  cudaGetDevice(&dev);
  static std::atomic<int> cache[64] = {};
  if (dev >= 0 && dev < 64 && (n = cache[dev].load(std::memory_order_relaxed)) > 0) return n;
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  if (n <= 0) n = 148;
  if (dev >= 0 && dev < 64) cache[dev].store(n, std::memory_order_relaxed);
  return n;
}

int gemm_prepare(GemmOp* op, const __half* A, int M, int K, const DevMatrix& Win, const float* bias, int epi,
                 void* out, int ldo, const QkvDst* qkv, const PatchSrc* patch) {
  // A quantised matrix loaded with a dequantised f16 copy runs on that copy
  // once there are at least 256 rows; without one, GEMMs of 256 rows or more
  // unpack it in the CTA-pair kernel's loader (each SM unpacks half of the
  // 256 x 64 weight tile of a 256 x 256 x 64 product) and smaller ones in
  // the single-CTA kernel's.
  DevMatrix W = Win;
  // a patch source (EPI_PATCH) comes with A, the unfolded patch matrix; the
  // epilogue places the rows and adds the positional table
  if (W.bmode != B_F16 && W.f16 && !patch && M >= 256) {
    W.bmode = B_F16;
    W.data = W.f16;
    W.scales = nullptr;
  }
  if (!op || !out || M < 1 || K < 64 || K % 64 != 0 || W.K != K || W.N < 1 || !W.data) return JEPA_B200_ERR_SHAPE;
  if (!A) return JEPA_B200_ERR_ARG;
  const int N = W.N;
  const int bn = N % 256 == 0 ? 256 : (N % 192 == 0 ? 192 : (N % 128 == 0 ? 128 : 0));
  if (!bn) return JEPA_B200_ERR_SHAPE;
  if (patch && W.bmode != B_F16) return JEPA_B200_ERR_UNSUPPORTED;
  if (W.bmode != B_F16 && !W.scales) return JEPA_B200_ERR_ARG;
  if ((epi == EPI_F16 || epi == EPI_GELU_F16 || epi == EPI_RESID_F32 || epi == EPI_F32) && ldo < N)
    return JEPA_B200_ERR_SHAPE;
  memset(op, 0, sizeof(*op));
  op->bn = bn;
  op->bmode = W.bmode;
  op->bf16 = W.bf16;  // the model's 16-bit type: A, the unpacked weights and 16-bit outputs
  op->gather = 0;
  GemmParams& p = op->p;
  p.M = M;
  p.N = N;
  p.K = K;
  p.m_tiles = (M + 127) / 128;
  p.n_tiles = N / bn;
  p.bias = bias;
  p.epi = epi;
  p.out = out;
  p.ldo = ldo;
  if (qkv) p.qkv = *qkv;
  if (patch) p.patch = *patch;
  p.bq = W.bmode != B_F16 ? W.data : nullptr;
  p.bscale = W.scales;
  {
    const uint64_t dims[2] = {static_cast<uint64_t>(K), static_cast<uint64_t>(M)};
    const uint64_t str[1] = {static_cast<uint64_t>(K) * 2};
    const uint32_t box[2] = {64, 128};
    if (!make_tmap_f16(&op->tmA, A, 2, dims, str, box)) return JEPA_B200_ERR_CUDA;
  }
  // TMA epilogue: f32 outputs and residual adds in 32-column chunks, f16
  // outputs in 64-column chunks (two per warp-half of the tile)
  if (epi == EPI_F32 || epi == EPI_RESID_F32) {
    if (!make_tmap_2d(&op->tmC, out, 4, static_cast<uint64_t>(ldo), static_cast<uint64_t>(M),
                      static_cast<uint64_t>(ldo) * 4, 32, 32))
      return JEPA_B200_ERR_CUDA;
    p.tma_epi = 1;
  } else if ((epi == EPI_F16 || epi == EPI_GELU_F16) && (bn / 64) % 2 == 0) {
    if (!make_tmap_2d(&op->tmC, out, 2, static_cast<uint64_t>(ldo), static_cast<uint64_t>(M),
                      static_cast<uint64_t>(ldo) * 2, 64, 32))
      return JEPA_B200_ERR_CUDA;
    p.tma_epi = 1;
  }
  // QKV epilogue: Q and K as [B*h, N, 64] maps, 32 token rows per store
  if (epi == EPI_QKV && qkv && (bn / 64) % 2 == 0 && qkv->ntok > 0 && M % qkv->ntok == 0 && qkv->dim % 64 == 0 &&
      qkv->head_dim == 64) {
    const uint64_t BHn = static_cast<uint64_t>(M / qkv->ntok) * qkv->heads;
    const uint64_t dims[3] = {64, static_cast<uint64_t>(qkv->ntok), BHn};
    const uint64_t str[2] = {128, static_cast<uint64_t>(qkv->ntok) * 128};
    const uint32_t box[3] = {64, 32, 1};
    // a map is built for a missing destination too (on the other one's
    // address); the epilogue never stores through it
    const __half* qb = qkv->q ? qkv->q : qkv->k;
    const __half* kb = qkv->k ? qkv->k : qkv->q;
    if (qb && kb) {
      if (!make_tmap_f16(&op->tmC, qb, 3, dims, str, box) || !make_tmap_f16(&op->tmC2, kb, 3, dims, str, box))
        return JEPA_B200_ERR_CUDA;
      p.tma_epi = 1;
    }
  }
  // at least two 128-row blocks: the CTA-pair kernel (quantised weights need
  // a scale table whose rows TMA can address: 8-scale groups, 16-byte rows)
  op->pair = (M >= 256 && (W.bmode == B_F16 || (W.scales_pad && W.sc_ld % 8 == 0))) ? 1 : 0;
  if (W.bmode == B_F16) {
    const uint64_t dims[2] = {static_cast<uint64_t>(K), static_cast<uint64_t>(N)};
    const uint64_t str[1] = {static_cast<uint64_t>(K) * 2};
    const uint32_t box[2] = {64, static_cast<uint32_t>(op->pair ? bn / 2 : bn)};
    if (!make_tmap_f16(&op->tmB, W.data, 2, dims, str, box)) return JEPA_B200_ERR_CUDA;
  } else if (op->pair) {
    // codes [N, K] bytes (q8_0) or [N, K/2] (q4_0): one K block of BN/2 rows
    // per load; scales [N, sc_ld] f16: the 8-scale group holding the K block's two
    const uint64_t row = W.bmode == B_Q8 ? static_cast<uint64_t>(K) : static_cast<uint64_t>(K) / 2;
    if (!make_tmap_plain(&op->tmB, W.data, CU_TENSOR_MAP_DATA_TYPE_UINT8, row, static_cast<uint64_t>(N), row,
                         W.bmode == B_Q8 ? 64u : 32u, static_cast<uint32_t>(bn / 2)))
      return JEPA_B200_ERR_CUDA;
    if (!make_tmap_plain(&op->tmS, W.scales_pad, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, static_cast<uint64_t>(W.sc_ld),
                         static_cast<uint64_t>(N), static_cast<uint64_t>(W.sc_ld) * 2, 8u,
                         static_cast<uint32_t>(bn / 2)))
      return JEPA_B200_ERR_CUDA;
  }
  if (op->pair) {
    const int cluster_tiles = ((M + 255) / 256) * p.n_tiles;
    op->grid = 2 * std::min(cluster_tiles, num_sms() / 2);
    op->smem = bn == 256 ? Gemm2Cfg<256, B_F16>::SMEM : (bn == 192 ? Gemm2Cfg<192, B_F16>::SMEM : Gemm2Cfg<128, B_F16>::SMEM);
  } else {
    op->grid = std::min(p.m_tiles * p.n_tiles, num_sms());
    op->smem = bn == 256 ? GemmCfg<256>::SMEM : (bn == 192 ? GemmCfg<192>::SMEM : GemmCfg<128>::SMEM);
  }
  return JEPA_B200_OK;
}

template <int BN, int BMODE, bool ROPE, bool BF>
static int launch_impl(const GemmOp& op, cudaStream_t st) {
  auto kern = gemm_tc_kernel<BN, BMODE, ROPE, BF>;
  static std::atomic<unsigned long long> attr_done{0};
  if (!smem_attr_once(attr_done, kern, GemmCfg<BN>::SMEM)) return JEPA_B200_ERR_CUDA;
  constexpr int threads = BMODE != B_F16 ? 448 : 320;
  if (launch_pdl(kern, dim3(op.grid), dim3(threads), GemmCfg<BN>::SMEM, st, 1, op.tmA, op.tmB, op.tmC, op.tmC2, op.p) !=
      cudaSuccess)
    return JEPA_B200_ERR_CUDA;
  return JEPA_B200_OK;
}

template <int BN, bool ROPE, int BMODE, bool BF>
static int launch_pair(const GemmOp& op, cudaStream_t st) {
  using C = Gemm2Cfg<BN, BMODE>;
  auto kern = gemm_pair_kernel<BN, ROPE, BMODE, BF>;
  static std::atomic<unsigned long long> attr_done{0};
  if (!smem_attr_once(attr_done, kern, C::SMEM)) return JEPA_B200_ERR_CUDA;
  if (launch_pdl(kern, dim3(op.grid), dim3(C::THREADS), C::SMEM, st, 2, op.tmA, op.tmB, op.tmC, op.tmC2, op.tmS,
                 op.p) != cudaSuccess)
    return JEPA_B200_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? JEPA_B200_OK : JEPA_B200_ERR_CUDA;
}

// Every instance is selected here from the op: tile width, weight format,
// rotary q / k, 16-bit activation type.
template <bool BF>
static int launch_typed(const GemmOp& op, cudaStream_t st) {
  // rotary q / k only in the QKV GEMMs of a rotary model: their own instances,
  // so that the others carry no rotation code
  const bool rope = op.p.epi == EPI_QKV && op.p.qkv.rope;
#define JB_PAIR(BNV)                                                                                              \
  switch (op.bmode) {                                                                                             \
    case B_Q8: return rope ? launch_pair<BNV, true, B_Q8, BF>(op, st) : launch_pair<BNV, false, B_Q8, BF>(op, st); \
    case B_Q4: return rope ? launch_pair<BNV, true, B_Q4, BF>(op, st) : launch_pair<BNV, false, B_Q4, BF>(op, st); \
    default: return rope ? launch_pair<BNV, true, B_F16, BF>(op, st) : launch_pair<BNV, false, B_F16, BF>(op, st); \
  }
#define JB_SINGLE(BNV)                                                                                              \
  switch (op.bmode) {                                                                                               \
    case B_Q8: return rope ? launch_impl<BNV, B_Q8, true, BF>(op, st) : launch_impl<BNV, B_Q8, false, BF>(op, st); \
    case B_Q4: return rope ? launch_impl<BNV, B_Q4, true, BF>(op, st) : launch_impl<BNV, B_Q4, false, BF>(op, st); \
    default: return rope ? launch_impl<BNV, B_F16, true, BF>(op, st) : launch_impl<BNV, B_F16, false, BF>(op, st); \
  }
  if (op.pair) {
    switch (op.bn) {
      case 256: JB_PAIR(256)
      case 192: JB_PAIR(192)
      default: JB_PAIR(128)
    }
  }
  switch (op.bn) {
    case 256: JB_SINGLE(256)
    case 192: JB_SINGLE(192)
    case 128: JB_SINGLE(128)
    default: return JEPA_B200_ERR_SHAPE;
  }
#undef JB_SINGLE
#undef JB_PAIR
}

int gemm_launch(const GemmOp& op_in, cudaStream_t st, DevErr* err, unsigned long long timeout_ns) {
  GemmOp op = op_in;
  op.p.err = err;
  op.p.timeout_ns = timeout_ns;
  return op.bf16 ? launch_typed<true>(op, st) : launch_typed<false>(op, st);
}

}  // namespace jb
