// Host-side declarations shared by the translation units of libjepa_b200.
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <atomic>

#include "../../include/jepa_b200.h"
#include "common.cuh"

namespace jb {

enum Epi { EPI_F16 = 0, EPI_GELU_F16 = 1, EPI_RESID_F32 = 2, EPI_F32 = 3, EPI_QKV = 4, EPI_PATCH = 5 };
enum BMode { B_F16 = 0, B_Q8 = 1, B_Q4 = 2 };

constexpr unsigned long long kDefaultTimeoutNs = 4000000000ull;

// A weight matrix [N, K] on the device in the GEMM's layout.
struct DevMatrix {
  int bmode = B_F16;  // B_F16 | B_Q8 | B_Q4
  int N = 0, K = 0;   // K: row length as stored (f16: padded to 64 with zeros)
  void* data = nullptr;       // f16 [N, K] | int8 [N, K] | nibble bytes [N, K/2]
  __half* scales = nullptr;   // fp16 [N, K/32] for quantised matrices
  // the same scales in rows of sc_ld (a multiple of 8) entries, zero-padded,
  // for the CTA-pair kernel's TMA-staged loader (may alias scales)
  __half* scales_pad = nullptr;
  int sc_ld = 0;
  // quantised matrices: the same values dequantised once to f16 [N, K] (each
  // q * d or (q - 8) * d rounded once, as the in-loader unpack rounds them),
  // used by GEMMs with M >= 256 rows, where the unpack in the loader cannot
  // keep pace with the tensor cores; null where absent
  __half* f16 = nullptr;
  // 16-bit data (B_F16, and the f16 copy) holds bf16 values instead of f16
  int bf16 = 0;
};

// Destination of the QKV scatter epilogue.
struct QkvDst {
  __half* q = nullptr;
  __half* k = nullptr;
  __half* vt = nullptr;
  int ntok = 0, heads = 0, npad = 0, first_part = 0, dim = 0;
  // dims per head: 64, or 32 (written to dims 0..31 of the 64-dim rows of Q,
  // K and V^T, whose dims 32..63 hold zeros)
  int head_dim = 64;
  // 3-D rotary positions of q and k (null: none): (cos, sin) [3 axes][kRopeMaxPos][10]
  const float2* rope = nullptr;
  int rope_ppf = 0, rope_pw = 0;  // patches per slot, per patch row
};

// Positions per axis the rotary table holds (slots, patch rows, patch columns).
constexpr int kRopeMaxPos = 64;

// Source geometry of the patch-embed (the patch matrix and the GEMM epilogue).
struct PatchSrc {
  const float* pixels = nullptr;
  int T = 0, H = 0, W = 0, patch = 0, tubelet = 0;
  int n_patches = 0;   // per clip
  int k_real = 0;      // 3 * kt * p * p
  const float* pos = nullptr;  // [ntok, D]
  int ntok = 0, has_cls = 0;
};

struct GemmParams {
  int M, N, K;
  int tma_epi;  // 1: the epilogue stages 32-row chunks in shared memory and writes them with TMA
  int m_tiles, n_tiles;
  const float* bias;
  int epi;
  void* out;
  int ldo;
  QkvDst qkv;
  PatchSrc patch;
  const void* bq;           // quantised weights
  const __half* bscale;
  DevErr* err;
  unsigned long long timeout_ns;
};

// Everything one GEMM launch needs, built once and replayed.
struct GemmOp {
  CUtensorMap tmA;
  CUtensorMap tmB;
  CUtensorMap tmC;   // output map of the TMA epilogue (Q for the QKV epilogue)
  CUtensorMap tmC2;  // K map of the QKV epilogue
  CUtensorMap tmS;   // quantised weights in the CTA-pair kernel: scale groups (tmB: the codes)
  GemmParams p;
  int bn = 0, bmode = 0, gather = 0, grid = 0, smem = 0;
  int pair = 0;  // 1: CTA-pair kernel (tcgen05 cta_group::2, 256-row tiles)
  int bf16 = 0;  // A, the weights' 16-bit form and 16-bit outputs in bf16 instead of f16
};

// Build a GEMM op.  A: f16 [M, K] (ignored when patch != nullptr: the patch
// pixels are gathered instead).  Returns a jepa_b200_status.
int gemm_prepare(GemmOp* op, const __half* A, int M, int K, const DevMatrix& W, const float* bias, int epi,
                 void* out, int ldo, const QkvDst* qkv, const PatchSrc* patch);
int gemm_launch(const GemmOp& op, cudaStream_t st, DevErr* err, unsigned long long timeout_ns);

struct AttnParams {
  int N, heads, n_q_tiles, mask, has_cls, ppf;
  int cls_separate;  // block-causal with CLS: row 0 computed apart from query tile 0
  int cls_in_pair;   // ... as the second query tile of the last pair (odd tile count), else in a CTA of its own
  int cls_tail;      // one tile per CTA: ... as padding row N of the last query tile (N % 128 != 0)
  const __half* q;   // Q [B*h, N, 64] (the CLS query row copied into that padding row)
  float scale_log2;
  __half* out;
  int ldo;
  int dv;            // dims per head written to out (32 or 64)
  DevErr* err;
  unsigned long long timeout_ns;
};

struct AttnOp {
  CUtensorMap tmQ, tmK, tmV;
  AttnParams p;
  int bf16 = 0;  // Q, K, V^T, P and the output in bf16 instead of f16
  const __half* q = nullptr;
  const __half* k = nullptr;
  const __half* vt = nullptr;
  int npad = 0;
  int B = 0, smem = 0;
};

// head_dim 64, or 32 (Q, K, V^T still [.., 64] rows with dims 32..63 zero;
// out [B*ntok, heads*head_dim])
int attn_prepare(AttnOp* op, const __half* q, const __half* k, const __half* vt, int B, int heads, int ntok,
                 int npad, int mask, int has_cls, int ppf, __half* out, int head_dim = 64);
int attn_launch(const AttnOp& op, cudaStream_t st, DevErr* err, unsigned long long timeout_ns);

// LayerNorm: rows of D f32 -> f16 or f32; input row r*in_stride.
// 16-bit outputs (out_f16) are bf16 when bf16 is set.
int launch_layernorm(const float* x, int rows, int D, long long in_stride, const float* g, const float* b,
                     float eps, void* out, bool out_f16, cudaStream_t st, bool bf16 = false);
// LayerNorm of `rows` rows where output row r reads input row
// (r / grp) * grp_stride + grp_off + r % grp (a block of grp rows out of
// every grp_stride).
int launch_layernorm_rows(const float* x, int rows, int D, int grp, long long grp_stride, int grp_off, const float* g,
                          const float* b, float eps, void* out, bool out_f16, cudaStream_t st, bool bf16 = false);
// Masked predictor input: a[b*nsel + i] = f16(tokens[b, idx[i]]) (device
// idx); x = [e rows + pos[ctx] | mask + pos[tgt]] per clip.
int launch_gather_rows_f16(const float* tokens, const int* idx, int B, int ntok, int nsel, int D, __half* a,
                           cudaStream_t st, bool bf16 = false);
int launch_pred_assemble(const float* e, const float* mask, const float* pos, const int* ctx, const int* tgt, int B,
                         int nctx, int ntgt, int D, float* x, cudaStream_t st);
// Write the CLS rows x[b*ntok + 0] = cls + pos[0].
int launch_cls_rows(float* x, int B, int ntok, int D, const float* cls, const float* pos, cudaStream_t st);
int launch_mean_pool(const float* y, int B, int ntok, int D, int first, float* partial, float* out,
                     cudaStream_t st);
int mean_pool_partial_floats(int B, int D);
int launch_repack(int bmode, const uint8_t* blocks, int N, int K, void* qs, __half* scales, cudaStream_t st);
// f16 [N, K] from repacked q8_0 / q4_0 quants and scales (DevMatrix::f16).
int launch_dequant_f16(int bmode, const void* qs, const __half* scales, int N, int K, __half* out, cudaStream_t st,
                       bool bf16 = false);
int launch_gemv(const float* x, int M, int K, const DevMatrix& W, const float* bias, int epi, const float* resid,
                long long resid_stride, float* y, cudaStream_t st);
int launch_xattn_1q(const float* q, const __half* k, const __half* vt, int B, int heads, int ntok, int npad,
                    float* out, cudaStream_t st, bool bf16 = false);

// Driver entry point for tensor maps (resolved once through the runtime).
bool make_tmap_f16(CUtensorMap* m, const void* base, int rank, const uint64_t* dims, const uint64_t* strides_bytes,
                   const uint32_t* box);
// 2-D map with 128-byte swizzle of f16 (esize 2) or f32 (esize 4) elements.
bool make_tmap_2d(CUtensorMap* m, const void* base, int esize, uint64_t cols, uint64_t rows, uint64_t row_bytes,
                  uint32_t box_cols, uint32_t box_rows);

int num_sms();

// Raise a kernel's dynamic shared-memory limit to `bytes` once per device.
// `done` holds one bit per device (0..63); the entry points may be called
// from several host threads, so the bit is read and set atomically (two
// threads that race both set the attribute, which is harmless).
template <typename Kern>
inline bool smem_attr_once(std::atomic<unsigned long long>& done, Kern kern, int bytes) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  const unsigned long long bit = dev >= 0 && dev < 64 ? (1ull << dev) : 0ull;
  if (bit && (done.load(std::memory_order_acquire) & bit)) return true;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess) return false;
  if (bit) done.fetch_or(bit, std::memory_order_release);
  return true;
}

// Launch with programmatic stream serialization (and, cluster_x > 1, thread
// block clusters of cluster_x CTAs): the kernel calls pdl_wait() before
// touching what earlier kernels in the stream wrote.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                              int cluster_x, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  int n = 0;
  attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[n].val.programmaticStreamSerializationAllowed = 1;
  ++n;
  if (cluster_x > 1) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = cluster_x;
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, kern, args...);
}

}  // namespace jb
