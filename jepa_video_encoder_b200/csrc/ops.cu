// Single-kernel entry points of the C ABI: each validates its arguments on
// the host and enqueues exactly the kernel the forward pass uses.
#include <string.h>

#include <mutex>

#include "internal.h"
#include "patchify.h"

using namespace jb;

namespace {

unsigned long long g_timeout_ns = kDefaultTimeoutNs;
std::mutex g_err_mu;
DevErr* g_err[64] = {nullptr};

// The per-device error word of the op entry points (allocated on first use).
DevErr* op_err() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lk(g_err_mu);
  if (!g_err[dev]) {
    void* p = nullptr;
    if (cudaMalloc(&p, sizeof(DevErr)) != cudaSuccess) return nullptr;
    if (cudaMemset(p, 0, sizeof(DevErr)) != cudaSuccess) {
      cudaFree(p);
      return nullptr;
    }
    g_err[dev] = static_cast<DevErr*>(p);
  }
  return g_err[dev];
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int bmode_of(int dtype) {
  switch (dtype) {
    case JEPA_B200_F16: return B_F16;
    case JEPA_B200_Q8_0: return B_Q8;
    case JEPA_B200_Q4_0: return B_Q4;
    default: return -1;
  }
}

int make_matrix(DevMatrix* W, const void* w, const void* scales, int dtype, int N, int K) {
  const int bm = bmode_of(dtype);
  if (bm < 0) return JEPA_B200_ERR_DTYPE;
  if (!w || (bm != B_F16 && !scales)) return JEPA_B200_ERR_ARG;
  if (!aligned16(w)) return JEPA_B200_ERR_ARG;
  W->bmode = bm;
  W->N = N;
  W->K = K;
  W->data = const_cast<void*>(w);
  W->scales = static_cast<__half*>(const_cast<void*>(scales));
  // the caller's [N, K/32] scales serve the CTA-pair kernel's staged loader
  // when their rows are whole 16-byte groups (K a multiple of 256) and 16-byte aligned
  if (bm != B_F16 && (K / 32) % 8 == 0 && aligned16(scales)) {
    W->scales_pad = W->scales;
    W->sc_ld = K / 32;
  }
  return JEPA_B200_OK;
}

}  // namespace

extern "C" {

void jepa_b200_op_set_timeout_ns(unsigned long long ns) { g_timeout_ns = ns; }

int jepa_b200_op_sync_status(void* stream) {
  DevErr* e = op_err();
  if (!e) return JEPA_B200_ERR_CUDA;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return JEPA_B200_ERR_CUDA;
  DevErr h{0, 0};
  if (cudaMemcpy(&h, e, sizeof(h), cudaMemcpyDeviceToHost) != cudaSuccess) return JEPA_B200_ERR_CUDA;
  if (h.code != DERR_NONE) {
    cudaMemset(e, 0, sizeof(DevErr));
    return h.code == DERR_TIMEOUT ? JEPA_B200_ERR_TIMEOUT : JEPA_B200_ERR_CUDA;
  }
  return JEPA_B200_OK;
}

int jepa_b200_op_layernorm(const float* x, int rows, int D, int in_row_stride, const float* gamma,
                           const float* beta, float eps, void* out, int out_dtype, void* stream) {
  if (out_dtype != JEPA_B200_F16 && out_dtype != JEPA_B200_F32) return JEPA_B200_ERR_DTYPE;
  if (!aligned16(x) || !aligned16(out) || !aligned16(gamma) || !aligned16(beta)) return JEPA_B200_ERR_ARG;
  if (!(eps > 0.0f)) return JEPA_B200_ERR_ARG;
  return launch_layernorm(x, rows, D, in_row_stride, gamma, beta, eps, out, out_dtype == JEPA_B200_F16,
                          static_cast<cudaStream_t>(stream));
}

int jepa_b200_op_repack(int dtype, const void* blocks, int N, int K, void* qs, void* scales, void* stream) {
  const int bm = bmode_of(dtype);
  if (bm != B_Q8 && bm != B_Q4) return JEPA_B200_ERR_DTYPE;
  return launch_repack(bm, static_cast<const uint8_t*>(blocks), N, K, qs, static_cast<__half*>(scales),
                       static_cast<cudaStream_t>(stream));
}

int jepa_b200_op_dequant_f16(int dtype, const void* qs, const void* scales, int N, int K, void* out, void* stream) {
  const int bm = bmode_of(dtype);
  if (bm != B_Q8 && bm != B_Q4) return JEPA_B200_ERR_DTYPE;
  if (!qs || !scales || !out || !aligned16(out)) return JEPA_B200_ERR_ARG;
  return launch_dequant_f16(bm, qs, static_cast<const __half*>(scales), N, K, static_cast<__half*>(out),
                            static_cast<cudaStream_t>(stream));
}

int jepa_b200_op_linear(const void* A, int M, int K, const void* w, const void* w_scales, int w_dtype, int N,
                        const float* bias, int epilogue, void* out, int ldo, void* stream) {
  if (!A || !out) return JEPA_B200_ERR_ARG;
  if (epilogue < JEPA_B200_EPI_F16 || epilogue > JEPA_B200_EPI_F32) return JEPA_B200_ERR_ARG;
  if (!aligned16(A) || !aligned16(out) || (bias && !aligned16(bias)) || ldo % 8 != 0) return JEPA_B200_ERR_ARG;
  DevMatrix W;
  int s = make_matrix(&W, w, w_scales, w_dtype, N, K);
  if (s) return s;
  DevErr* e = op_err();
  if (!e) return JEPA_B200_ERR_CUDA;
  GemmOp op;
  if ((s = gemm_prepare(&op, static_cast<const __half*>(A), M, K, W, bias, epilogue, out, ldo, nullptr, nullptr)))
    return s;
  return gemm_launch(op, static_cast<cudaStream_t>(stream), e, g_timeout_ns);
}

int jepa_b200_op_linear_qkv(const void* A, int M, int K, const void* w, const void* w_scales, int w_dtype, int N,
                            const float* bias, int ntok, int heads, int npad, int first_part, void* q, void* k,
                            void* vt, void* stream) {
  if (!A || heads < 1 || ntok < 1 || first_part < 0 || first_part > 2) return JEPA_B200_ERR_ARG;
  const int D = 64 * heads;
  if (N % D != 0 || N / D + first_part > 3 || M % ntok != 0 || npad < ntok || npad % 128 != 0)
    return JEPA_B200_ERR_SHAPE;
  if (!aligned16(A) || (bias && !aligned16(bias)) || (q && !aligned16(q)) || (k && !aligned16(k)))
    return JEPA_B200_ERR_ARG;
  DevMatrix W;
  int s = make_matrix(&W, w, w_scales, w_dtype, N, K);
  if (s) return s;
  DevErr* e = op_err();
  if (!e) return JEPA_B200_ERR_CUDA;
  QkvDst qd;
  qd.q = static_cast<__half*>(q);
  qd.k = static_cast<__half*>(k);
  qd.vt = static_cast<__half*>(vt);
  qd.ntok = ntok;
  qd.heads = heads;
  qd.npad = npad;
  qd.first_part = first_part;
  qd.dim = D;
  void* anyout = q ? q : (k ? k : vt);
  if (!anyout) return JEPA_B200_ERR_ARG;
  GemmOp op;
  if ((s = gemm_prepare(&op, static_cast<const __half*>(A), M, K, W, bias, EPI_QKV, anyout, N, &qd, nullptr)))
    return s;
  return gemm_launch(op, static_cast<cudaStream_t>(stream), e, g_timeout_ns);
}

int jepa_b200_op_attention(const void* q, const void* k, const void* vt, int B, int heads, int ntok, int npad,
                           int mask, int has_cls, int patches_per_slot, void* out, void* stream) {
  if (!aligned16(q) || !aligned16(k) || !aligned16(vt) || !aligned16(out)) return JEPA_B200_ERR_ARG;
  DevErr* e = op_err();
  if (!e) return JEPA_B200_ERR_CUDA;
  AttnOp op;
  int s = attn_prepare(&op, static_cast<const __half*>(q), static_cast<const __half*>(k),
                       static_cast<const __half*>(vt), B, heads, ntok, npad, mask, has_cls, patches_per_slot,
                       static_cast<__half*>(out));
  if (s) return s;
  return attn_launch(op, static_cast<cudaStream_t>(stream), e, g_timeout_ns);
}

int jepa_b200_op_patch_embed(const float* pixels, int B, int T, int H, int W, int patch, int tubelet,
                             const void* w_pe, int D, const float* bias, const float* pos, const float* cls,
                             int has_cls, float* x, void* stream) {
  if (!pixels || !w_pe || !pos || !x || (has_cls && !cls)) return JEPA_B200_ERR_ARG;
  if (B < 1 || patch < 1 || tubelet < 1 || T < tubelet || T % tubelet || H % patch || W % patch || H < patch ||
      W < patch || D < 64 || D % 32 != 0)
    return JEPA_B200_ERR_SHAPE;
  if (!aligned16(x) || !aligned16(pos) || (bias && !aligned16(bias))) return JEPA_B200_ERR_ARG;
  // the limits of the model loader: K = 3 * kt * p^2 <= 32768, B * ntok * 4096 < 2^31
  if (D > 4096 || 3ll * tubelet * patch * patch > 32768 ||
      static_cast<long long>(B) * ((static_cast<long long>(T / tubelet) * (H / patch) * (W / patch)) + 1) >
          (1ll << 31) / 4096)
    return JEPA_B200_ERR_SHAPE;
  const int k_real = 3 * tubelet * patch * patch;
  const int kpad = (k_real + 63) / 64 * 64;
  const int n_patches = (T / tubelet) * (H / patch) * (W / patch);
  const int ntok = n_patches + (has_cls ? 1 : 0);
  DevMatrix Wm;
  int s = make_matrix(&Wm, w_pe, nullptr, JEPA_B200_F16, D, kpad);
  if (s) return s;
  DevErr* e = op_err();
  if (!e) return JEPA_B200_ERR_CUDA;
  PatchSrc ps;
  ps.pixels = pixels;
  ps.T = T;
  ps.H = H;
  ps.W = W;
  ps.patch = patch;
  ps.tubelet = tubelet;
  ps.n_patches = n_patches;
  ps.k_real = k_real;
  ps.pos = pos;
  ps.ntok = ntok;
  ps.has_cls = has_cls ? 1 : 0;
  // the unfolded patch matrix goes to a per-device scratch buffer that grows
  // on demand (growing waits for the device to be idle)
  static std::mutex mu;
  static void* scratch[64] = {nullptr};
  static size_t scratch_bytes[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return JEPA_B200_ERR_CUDA;
  const size_t need = static_cast<size_t>(B) * n_patches * kpad * 2;
  void* a = nullptr;
  {
    std::lock_guard<std::mutex> lk(mu);
    if (scratch_bytes[dev] < need) {
      cudaDeviceSynchronize();
      if (scratch[dev]) cudaFree(scratch[dev]);
      scratch[dev] = nullptr;
      scratch_bytes[dev] = 0;
      if (cudaMalloc(&scratch[dev], need) != cudaSuccess) return JEPA_B200_ERR_CUDA;
      scratch_bytes[dev] = need;
    }
    a = scratch[dev];
  }
  GemmOp op;
  if ((s = gemm_prepare(&op, static_cast<const __half*>(a), B * n_patches, kpad, Wm, bias, EPI_PATCH, x, D, nullptr,
                        &ps)))
    return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if ((s = launch_patchify(pixels, ps, B, kpad, a, st, false))) return s;
  if ((s = gemm_launch(op, st, e, g_timeout_ns))) return s;
  if (has_cls) return launch_cls_rows(x, B, ntok, D, cls, pos, st);
  return JEPA_B200_OK;
}

int jepa_b200_op_gemv(const float* x, int M, int K, const void* w, const void* w_scales, int w_dtype, int N,
                      const float* bias, int epi, const float* resid, int resid_row_stride, float* y, void* stream) {
  if (epi < 0 || epi > 2 || M > 64) return JEPA_B200_ERR_ARG;
  DevMatrix W;
  int s = make_matrix(&W, w, w_scales, w_dtype, N, K);
  if (s) return s;
  return launch_gemv(x, M, K, W, bias, epi, resid, resid_row_stride, y, static_cast<cudaStream_t>(stream));
}

int jepa_b200_op_xattn_1q(const float* q, const void* k, const void* vt, int B, int heads, int ntok, int npad,
                          float* out, void* stream) {
  if (!aligned16(k)) return JEPA_B200_ERR_ARG;
  return launch_xattn_1q(q, static_cast<const __half*>(k), static_cast<const __half*>(vt), B, heads, ntok, npad, out,
                         static_cast<cudaStream_t>(stream));
}

int jepa_b200_op_mean_pool(const float* y, int B, int ntok, int D, int first, float* out, void* stream) {
  if (!y || !out) return JEPA_B200_ERR_ARG;
  if (B < 1 || D < 1) return JEPA_B200_ERR_SHAPE;
  // partial column sums go to a per-device scratch buffer that grows on demand
  static std::mutex mu;
  static float* scratch[64] = {nullptr};
  static size_t scratch_n[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return JEPA_B200_ERR_CUDA;
  const size_t need = static_cast<size_t>(mean_pool_partial_floats(B, D));
  {
    std::lock_guard<std::mutex> lk(mu);
    if (scratch_n[dev] < need) {
      cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
      if (scratch[dev]) cudaFree(scratch[dev]);
      scratch[dev] = nullptr;
      scratch_n[dev] = 0;
      if (cudaMalloc(&scratch[dev], need * 4) != cudaSuccess) return JEPA_B200_ERR_CUDA;
      scratch_n[dev] = need;
    }
  }
  return launch_mean_pool(y, B, ntok, D, first, scratch[dev], out, static_cast<cudaStream_t>(stream));
}

}  // extern "C"
