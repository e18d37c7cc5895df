// Host runtime of the JEPA ViT encoder forward: weight loading from a tensor
// table, the device workspace, and the fixed kernel sequence of one forward
// pass (the C ABI calls of include/jepa_b200.h).
//
// Sequence of jepa_b200_encode (B clips, R = B * N token rows):
//   patch matrix, patch-embed GEMM (+ pos_embed) and the CLS rows   -> X f32 [R, D]
//   per block:  LN1 -> Y f16; QKV GEMM -> Q, K, V^T (head-major)
//               attention -> O f16 [R, D]; out GEMM: X += O Wo^T + bo
//               LN2 -> Y; up GEMM + GELU -> H f16 [R, 4D]; down GEMM: X += H Wd^T + bd
//   final LN -> full map / CLS rows / mean over patch tokens / attentive head.
// The block structure is the pre-LN block of the "Quantization" page ("The
// rule": ln1, attn_qkv, attn_out, ln2, ffn_up, ffn_down); the head follows
// "jepa.cpp -- measured benchmarks", "Attentive-pool head".
#include <string.h>

#include <algorithm>
#include <cmath>
#include <string>
#include <unordered_map>
#include <vector>

#include "internal.h"
#include "patchify.h"
#include "world_model.h"

using namespace jb;

namespace {

struct LayerW {
  float *ln1_g = nullptr, *ln1_b = nullptr, *ln2_g = nullptr, *ln2_b = nullptr;
  DevMatrix qkv, out, up, down;
  float *b_qkv = nullptr, *b_out = nullptr, *b_up = nullptr, *b_down = nullptr;
};

struct BlockOps {
  GemmOp qkv, out, up, down;
};

struct DeviceGuard {
  int prev = -1;
  explicit DeviceGuard(int dev) {
    cudaGetDevice(&prev);
    if (prev != dev) cudaSetDevice(dev);
  }
  ~DeviceGuard() {
    int cur = -1;
    cudaGetDevice(&cur);
    if (prev >= 0 && cur != prev) cudaSetDevice(prev);
  }
};

// The inputs a captured forward is bound to.
struct EncodeKey {
  const float* pixels = nullptr;
  const float* out = nullptr;
  int B = 0, pool = -1;
  unsigned long long timeout_ns = 0;
  bool operator==(const EncodeKey& o) const {
    return pixels == o.pixels && out == o.out && B == o.B && pool == o.pool && timeout_ns == o.timeout_ns;
  }
};

}  // namespace

struct jepa_b200_model {
  jepa_b200_config cfg{};
  int device = 0;
  int N = 0, Np = 0, ppf = 0, Kpe = 0, Kpe_pad = 0, npad = 0;
  DevMatrix pe;
  float *b_pe = nullptr, *pos = nullptr, *cls = nullptr;
  float2* rope = nullptr;  // rotary (cos, sin) table [3][kRopeMaxPos][10] (cfg.rope)
  std::vector<LayerW> enc, head;
  float *norm_g = nullptr, *norm_b = nullptr;
  bool has_head = false;
  float *query = nullptr, *lnkv_g = nullptr, *lnkv_b = nullptr, *ln2x_g = nullptr, *ln2x_b = nullptr;
  DevMatrix xq, xkv, xout, xup, xdown, hcls;
  float *b_xq = nullptr, *b_xkv = nullptr, *b_xout = nullptr, *b_xup = nullptr, *b_xdown = nullptr,
        *b_cls = nullptr;
  // masked predictor (cfg.pred_depth > 0)
  DevMatrix pembed, pproj;
  float *b_pembed = nullptr, *pmask = nullptr, *ppos = nullptr, *pnorm_g = nullptr, *pnorm_b = nullptr,
        *b_pproj = nullptr;
  std::vector<LayerW> pred;
  // LeWM world model (cfg.wm_depth > 0): the projector for POOL_LEWM and the
  // fused predictor's weight arenas and f32 vectors
  DevMatrix wproj0, wproj2;
  float *b_wproj0 = nullptr, *b_wproj2 = nullptr;
  WmArena wm;
  float *wm_w_act0 = nullptr, *wm_b_act0 = nullptr, *wm_b_act2 = nullptr, *wm_pos = nullptr;
  float *wm_b_ada = nullptr, *wm_b_qkv = nullptr, *wm_b_out = nullptr, *wm_b_up = nullptr, *wm_b_down = nullptr;
  float *wm_norm_g = nullptr, *wm_norm_b = nullptr, *wm_b_p0 = nullptr, *wm_b_p2 = nullptr;
  std::vector<void*> allocs;
  size_t weight_bytes = 0;

  // workspace for the largest B seen
  int ws_B = 0;   // clips the workspace holds
  int ops_B = 0;  // clips the prepared ops process
  float* X = nullptr;
  __half *Y = nullptr, *Q = nullptr, *Kb = nullptr, *Vt = nullptr, *O = nullptr, *H = nullptr;
  float *Yf = nullptr, *partial = nullptr;
  float *hq = nullptr, *hattn = nullptr, *hz = nullptr, *hzn = nullptr, *hu = nullptr;
  float* hp = nullptr;  // the LeWM projector's hidden rows [B, wm_proj_hidden]
  __half* Ape = nullptr;  // the unfolded patch matrix [B * Np, Kpe_pad] (patch-embed A operand)
  std::vector<void*> ws_allocs;
  std::vector<BlockOps> enc_ops, head_ops;
  GemmOp pe_op, kv_op;
  AttnOp attn_enc, attn_head;

  // predictor workspace, for up to pws_rows sequence rows (B * (n_ctx + n_tgt))
  // and the ops of the last (B, n_ctx, n_tgt, tokens, out)
  size_t pws_rows = 0, pws_ctx_rows = 0, pws_tgt_rows = 0, pws_vt = 0;
  float *pX = nullptr, *pE = nullptr;
  __half *pY = nullptr, *pQ = nullptr, *pK = nullptr, *pVt = nullptr, *pO = nullptr, *pH = nullptr, *pA = nullptr,
         *pT = nullptr;
  int *pidx = nullptr;  // device ctx_idx [N] then tgt_idx [N]
  std::vector<int> pidx_host;
  std::vector<void*> pws_allocs;
  int pops_B = 0, pops_ctx = 0, pops_tgt = 0, pops_Lpad = 0;
  const float* pops_tokens = nullptr;
  float* pops_out = nullptr;
  std::vector<BlockOps> pred_ops;
  GemmOp pembed_op, pproj_op;
  AttnOp pattn;

  float* stage_pix = nullptr;
  size_t stage_pix_bytes = 0;
  float* stage_out = nullptr;
  size_t stage_out_bytes = 0;

  DevErr* err = nullptr;
  cudaEvent_t ev0 = nullptr, ev1 = nullptr;
  bool have_timing = false;
  unsigned long long timeout_ns = kDefaultTimeoutNs;
  int launches = 0;

  // CUDA graph of the last forward, replayed while its inputs (pointers, B,
  // pool, wait bound) are unchanged; captured on a stream of the model's own
  bool use_graph = true;
  cudaStream_t cap_stream = nullptr;
  cudaGraphExec_t graph = nullptr;
  EncodeKey g_key, last_key;  // inputs of the captured graph; of the previous encode
  int g_launches = 0;

  // per-kernel timing (jepa_b200_set_profiling)
  bool prof = false;
  std::vector<cudaEvent_t> prof_events;
  size_t prof_used = 0;
  struct ProfRec {
    int cls;
    size_t e0, e1;
  };
  std::vector<ProfRec> prof_recs;
};

namespace {

typedef std::unordered_map<std::string, const jepa_b200_tensor*> TableMap;

bool is_retyped(const std::string& n) {
  static const char* suffixes[] = {"attn_qkv.weight",     "attn_out.weight",     "ffn_up.weight",
                                   "ffn_down.weight",     "head.xattn.q.weight", "head.xattn.k.weight",
                                   "head.xattn.v.weight", "head.xattn.out.weight", "head.cls.weight",
                                   "pred.embed.weight",   "pred.proj.weight",    "enc.proj.0.weight",
                                   "enc.proj.2.weight",   "pred.proj.0.weight",  "pred.proj.2.weight"};
  for (const char* s : suffixes) {
    const size_t L = strlen(s);
    if (n.size() >= L && n.compare(n.size() - L, L, s) == 0) return true;
  }
  return false;
}

int64_t numel(const jepa_b200_tensor* t) {
  int64_t n = 1;
  for (int i = 0; i < t->ndim; ++i) n *= t->shape[i];
  return n;
}

size_t expected_bytes(const jepa_b200_tensor* t) {
  const int64_t n = numel(t);
  switch (t->dtype) {
    case JEPA_B200_F32: return static_cast<size_t>(n) * 4;
    case JEPA_B200_F16: return static_cast<size_t>(n) * 2;
    case JEPA_B200_Q8_0: return static_cast<size_t>(n / 32) * 34;
    case JEPA_B200_Q4_0: return static_cast<size_t>(n / 32) * 18;
    default: return 0;
  }
}

struct Loader {
  jepa_b200_model* m;
  TableMap tab;
  int status = JEPA_B200_OK;

  bool dry = false;  // validate only: no device calls, no conversions

  void* dalloc(size_t bytes) {
    void* p = nullptr;
    if (status != JEPA_B200_OK) return nullptr;
    if (dry) return reinterpret_cast<void*>(static_cast<uintptr_t>(256));
    if (cudaMalloc(&p, bytes) != cudaSuccess) {
      status = JEPA_B200_ERR_CUDA;
      return nullptr;
    }
    m->allocs.push_back(p);
    m->weight_bytes += bytes;
    return p;
  }
  bool upload(void* dst, const void* src, size_t bytes) {
    if (status != JEPA_B200_OK) return false;
    if (dry) return true;
    if (cudaMemcpy(dst, src, bytes, cudaMemcpyHostToDevice) != cudaSuccess) {
      status = JEPA_B200_ERR_CUDA;
      return false;
    }
    return true;
  }
  const jepa_b200_tensor* get(const std::string& name, std::initializer_list<int64_t> shape) {
    if (status != JEPA_B200_OK) return nullptr;
    auto it = tab.find(name);
    if (it == tab.end()) {
      status = JEPA_B200_ERR_MISSING_TENSOR;
      return nullptr;
    }
    const jepa_b200_tensor* t = it->second;
    if (t->ndim != static_cast<int>(shape.size())) {
      status = JEPA_B200_ERR_SHAPE;
      return nullptr;
    }
    int i = 0;
    for (int64_t s : shape) {
      if (t->shape[i++] != s) {
        status = JEPA_B200_ERR_SHAPE;
        return nullptr;
      }
    }
    const bool quant = t->dtype == JEPA_B200_Q8_0 || t->dtype == JEPA_B200_Q4_0;
    if (t->dtype != JEPA_B200_F32 && t->dtype != JEPA_B200_F16 && !quant) {
      status = JEPA_B200_ERR_DTYPE;
      return nullptr;
    }
    if (quant && !is_retyped(name)) {
      status = JEPA_B200_ERR_DTYPE;
      return nullptr;
    }
    if (!t->data || t->nbytes != expected_bytes(t)) {
      status = t->data ? JEPA_B200_ERR_SHAPE : JEPA_B200_ERR_ARG;
      return nullptr;
    }
    return t;
  }
  // host values of an f32 / f16 tensor as float
  std::vector<float> host_floats(const jepa_b200_tensor* t) {
    const int64_t n = numel(t);
    if (dry) return std::vector<float>(static_cast<size_t>(n));
    std::vector<float> v(static_cast<size_t>(n));
    if (t->dtype == JEPA_B200_F32) {
      memcpy(v.data(), t->data, static_cast<size_t>(n) * 4);
    } else {
      const __half* h = static_cast<const __half*>(t->data);
      for (int64_t i = 0; i < n; ++i) v[static_cast<size_t>(i)] = __half2float(h[i]);
    }
    return v;
  }
  float* vec(const std::string& name, int64_t len) {
    const jepa_b200_tensor* t = get(name, {len});
    if (!t) return nullptr;
    if (t->dtype != JEPA_B200_F32 && t->dtype != JEPA_B200_F16) {
      status = JEPA_B200_ERR_DTYPE;
      return nullptr;
    }
    std::vector<float> v = host_floats(t);
    float* d = static_cast<float*>(dalloc(v.size() * 4));
    if (d) upload(d, v.data(), v.size() * 4);
    return d;
  }
  float* table2d(const std::string& name, int64_t rows, int64_t cols) {
    const jepa_b200_tensor* t = get(name, {rows, cols});
    if (!t) return nullptr;
    if (t->dtype != JEPA_B200_F32 && t->dtype != JEPA_B200_F16) {
      status = JEPA_B200_ERR_DTYPE;
      return nullptr;
    }
    std::vector<float> v = host_floats(t);
    float* d = static_cast<float*>(dalloc(v.size() * 4));
    if (d) upload(d, v.data(), v.size() * 4);
    return d;
  }
  // Matrix [N, K] from one or more tensors stacked along N (all one dtype).
  DevMatrix matrix(const std::vector<const jepa_b200_tensor*>& parts, int64_t K, int64_t Kpad) {
    DevMatrix M;
    if (status != JEPA_B200_OK) return M;
    int64_t N = 0;
    const int dt = parts[0]->dtype;
    for (auto* t : parts) {
      if (t->dtype != dt) {
        status = JEPA_B200_ERR_DTYPE;
        return M;
      }
      N += numel(t) / K;
    }
    M.N = static_cast<int>(N);
    M.K = static_cast<int>(Kpad);
    const bool quant = dt == JEPA_B200_Q8_0 || dt == JEPA_B200_Q4_0;
    if (quant && (K % 64 != 0 || Kpad != K)) {
      status = JEPA_B200_ERR_SHAPE;
      return M;
    }
    if (dry) {
      M.bmode = dt == JEPA_B200_Q8_0 ? B_Q8 : (dt == JEPA_B200_Q4_0 ? B_Q4 : B_F16);
      M.data = dalloc(1);
      M.scales = quant ? static_cast<__half*>(dalloc(1)) : nullptr;
      M.scales_pad = M.scales;
      M.sc_ld = static_cast<int>((K / 32 + 7) / 8 * 8);
      M.f16 = quant && m->cfg.quant_f16_copy ? static_cast<__half*>(dalloc(1)) : nullptr;
      return M;
    }
    const bool bf = m->cfg.act_bf16 != 0;
    M.bf16 = bf ? 1 : 0;
    if (dt == JEPA_B200_F32 || dt == JEPA_B200_F16) {
      // the 16-bit operand: each value rounded once to f16, or to bf16 in a
      // bf16 model (from the table's f32 or f16 value)
      std::vector<uint16_t> h(static_cast<size_t>(N * Kpad), 0);
      int64_t row = 0;
      for (auto* t : parts) {
        std::vector<float> v = host_floats(t);
        const int64_t rows = numel(t) / K;
        for (int64_t r = 0; r < rows; ++r)
          for (int64_t k = 0; k < K; ++k) {
            const float x = v[static_cast<size_t>(r * K + k)];
            h[static_cast<size_t>((row + r) * Kpad + k)] =
                bf ? __bfloat16_as_ushort(__float2bfloat16_rn(x)) : __half_as_ushort(__float2half_rn(x));
          }
        row += rows;
      }
      M.bmode = B_F16;
      M.data = dalloc(h.size() * 2);
      if (M.data) upload(M.data, h.data(), h.size() * 2);
      return M;
    }
    // quantised: split the blocks into quants and fp16 scales (byte moves)
    const bool q8 = dt == JEPA_B200_Q8_0;
    const int bsz = q8 ? 34 : 18, qb = q8 ? 32 : 16;
    const int64_t nblk = N * (K / 32);
    std::vector<uint8_t> qs(static_cast<size_t>(nblk * qb));
    std::vector<uint16_t> sc(static_cast<size_t>(nblk));
    int64_t bi = 0;
    for (auto* t : parts) {
      const uint8_t* src = static_cast<const uint8_t*>(t->data);
      const int64_t nb = numel(t) / 32;
      for (int64_t i = 0; i < nb; ++i, ++bi) {
        const uint8_t* b = src + i * bsz;
        sc[static_cast<size_t>(bi)] = static_cast<uint16_t>(b[0] | (b[1] << 8));
        memcpy(&qs[static_cast<size_t>(bi * qb)], b + 2, qb);
      }
    }
    M.bmode = q8 ? B_Q8 : B_Q4;
    M.data = dalloc(qs.size());
    M.scales = static_cast<__half*>(dalloc(sc.size() * 2));
    if (M.data) upload(M.data, qs.data(), qs.size());
    if (M.scales) upload(M.scales, sc.data(), sc.size() * 2);
    // the scales again in rows padded to whole 8-scale (16-byte) groups, for
    // the CTA-pair kernel's TMA-staged loader (the same array when K / 32 is
    // a multiple of 8)
    const int64_t kq = K / 32, ld = (kq + 7) / 8 * 8;
    M.sc_ld = static_cast<int>(ld);
    if (ld == kq) {
      M.scales_pad = M.scales;
    } else {
      std::vector<uint16_t> sp(static_cast<size_t>(N * ld), 0);
      for (int64_t n = 0; n < N; ++n)
        for (int64_t j = 0; j < kq; ++j) sp[static_cast<size_t>(n * ld + j)] = sc[static_cast<size_t>(n * kq + j)];
      M.scales_pad = static_cast<__half*>(dalloc(sp.size() * 2));
      if (M.scales_pad) upload(M.scales_pad, sp.data(), sp.size() * 2);
    }
    // on request, the dequantised f16 copy for the large-M GEMMs, made on the device
    if (m->cfg.quant_f16_copy) {
      M.f16 = static_cast<__half*>(dalloc(static_cast<size_t>(N * K) * 2));
      if (M.f16 && status == JEPA_B200_OK &&
          launch_dequant_f16(M.bmode, M.data, M.scales, M.N, M.K, M.f16, nullptr, bf) != JEPA_B200_OK)
        status = JEPA_B200_ERR_CUDA;
    }
    return M;
  }
  // One matrix [N, K] into rows row0 .. row0 + N - 1 of a 16-bit arena of
  // row length K: f32 / f16 values rounded once to f16 (bf16 in a bf16
  // model); q8_0 / q4_0 blocks uploaded and unpacked on the device to the
  // same values the GEMM loaders produce.
  void arena_put(void* arena, int64_t row0, const std::string& name, int64_t N, int64_t K) {
    const jepa_b200_tensor* t = get(name, {N, K});
    if (!t || dry || status != JEPA_B200_OK) return;
    uint8_t* dst = static_cast<uint8_t*>(arena) + static_cast<size_t>(row0 * K) * 2;
    const bool bf = m->cfg.act_bf16 != 0;
    if (t->dtype == JEPA_B200_F32 || t->dtype == JEPA_B200_F16) {
      std::vector<float> v = host_floats(t);
      std::vector<uint16_t> h(v.size());
      for (size_t i = 0; i < v.size(); ++i)
        h[i] = bf ? __bfloat16_as_ushort(__float2bfloat16_rn(v[i])) : __half_as_ushort(__float2half_rn(v[i]));
      upload(dst, h.data(), h.size() * 2);
      return;
    }
    DevMatrix Q = matrix({t}, K, K);
    if (status == JEPA_B200_OK &&
        launch_dequant_f16(Q.bmode, Q.data, Q.scales, static_cast<int>(N), static_cast<int>(K),
                           reinterpret_cast<__half*>(dst), nullptr, bf) != JEPA_B200_OK)
      status = JEPA_B200_ERR_CUDA;
  }
  // The per-block f32 vectors prefix<i>.suffix [len] of blocks 0..n-1, stacked.
  float* vec_stack(const std::string& prefix, const std::string& suffix, int n, int64_t len) {
    std::vector<float> all;
    for (int i = 0; i < n && status == JEPA_B200_OK; ++i) {
      const jepa_b200_tensor* t = get(prefix + std::to_string(i) + "." + suffix, {len});
      if (!t) return nullptr;
      if (t->dtype != JEPA_B200_F32 && t->dtype != JEPA_B200_F16) {
        status = JEPA_B200_ERR_DTYPE;
        return nullptr;
      }
      std::vector<float> v = host_floats(t);
      all.insert(all.end(), v.begin(), v.end());
    }
    if (status != JEPA_B200_OK) return nullptr;
    float* d = static_cast<float*>(dalloc(all.size() * 4));
    if (d) upload(d, all.data(), all.size() * 4);
    return d;
  }
  DevMatrix mat(const std::string& name, int64_t N, int64_t K) {
    const jepa_b200_tensor* t = get(name, {N, K});
    if (!t) return DevMatrix();
    return matrix({t}, K, K);
  }
  void block(LayerW& L, const std::string& p, int64_t D, int64_t Mh) {
    L.ln1_g = vec(p + "ln1.weight", D);
    L.ln1_b = vec(p + "ln1.bias", D);
    L.qkv = mat(p + "attn_qkv.weight", 3 * D, D);
    L.b_qkv = vec(p + "attn_qkv.bias", 3 * D);
    L.out = mat(p + "attn_out.weight", D, D);
    L.b_out = vec(p + "attn_out.bias", D);
    L.ln2_g = vec(p + "ln2.weight", D);
    L.ln2_b = vec(p + "ln2.bias", D);
    L.up = mat(p + "ffn_up.weight", Mh, D);
    L.b_up = vec(p + "ffn_up.bias", Mh);
    L.down = mat(p + "ffn_down.weight", D, Mh);
    L.b_down = vec(p + "ffn_down.bias", D);
  }
};

void free_list(std::vector<void*>& v) {
  for (void* p : v) cudaFree(p);
  v.clear();
}

int validate_config(const jepa_b200_config* c) {
  if (!c) return JEPA_B200_ERR_ARG;
  if (c->dim < 64 || c->heads < 1 || c->dim != 64 * c->heads || c->dim % 64 || c->depth < 0 || c->mlp < 64 ||
      c->mlp % 64)
    return JEPA_B200_ERR_SHAPE;
  if (c->patch < 1 || c->tubelet < 1 || c->img_h < c->patch || c->img_w < c->patch || c->img_h % c->patch ||
      c->img_w % c->patch || c->frames < c->tubelet || c->frames % c->tubelet)
    return JEPA_B200_ERR_SHAPE;
  if (c->mask != JEPA_B200_MASK_BIDIR && c->mask != JEPA_B200_MASK_BLOCK_CAUSAL) return JEPA_B200_ERR_ARG;
  if (c->dim > 4096 || c->mlp > 16384) return JEPA_B200_ERR_SHAPE;
  // one clip must fit the row limit of a call (B * N * 4096 < 2^31), and the
  // patch vector 3 * kt * p * p the patch-embed's K
  const long long tokens = static_cast<long long>(c->frames / c->tubelet) * (c->img_h / c->patch) *
                           (c->img_w / c->patch) + (c->has_cls ? 1 : 0);
  if (tokens > (1ll << 31) / 4096) return JEPA_B200_ERR_SHAPE;
  if (3ll * c->tubelet * c->patch * c->patch > 32768) return JEPA_B200_ERR_SHAPE;
  if (c->n_classes < 0 || c->head_sa_blocks < 0) return JEPA_B200_ERR_ARG;
  if (!(c->ln_eps > 0.0f)) return JEPA_B200_ERR_ARG;
  if (c->rope != 0 && c->rope != 1) return JEPA_B200_ERR_ARG;
  if (c->quant_f16_copy != 0 && c->quant_f16_copy != 1) return JEPA_B200_ERR_ARG;
  if (c->act_bf16 != 0 && c->act_bf16 != 1) return JEPA_B200_ERR_ARG;
  if (c->pred_depth < 0) return JEPA_B200_ERR_ARG;
  if (c->pred_depth > 0) {
    if (c->pred_dim < 64 || c->pred_dim % 64 || c->pred_dim > 4096 || c->pred_heads < 1 ||
        c->pred_dim % c->pred_heads || c->pred_mlp < 64 || c->pred_mlp % 64 || c->pred_mlp > 16384)
      return JEPA_B200_ERR_SHAPE;
    const int hd = c->pred_dim / c->pred_heads;
    if (hd != 32 && hd != 64) return JEPA_B200_ERR_SHAPE;
  }
  if (c->wm_depth < 0) return JEPA_B200_ERR_ARG;
  if (c->wm_depth > 0 && c->pred_depth > 0) return JEPA_B200_ERR_ARG;  // both name their tensors pred.*
  if (c->wm_depth > 0) {
    // the fused world-model kernel: state width at most 256 in heads of 64,
    // MLP and output widths at most 1024, at most 32 frames a window
    if (c->dim > 256 || c->wm_heads < 1 || c->dim != 64 * c->wm_heads || c->wm_mlp < 64 || c->wm_mlp % 64 ||
        c->wm_mlp > 1024 || c->wm_pred_hidden < 64 || c->wm_pred_hidden % 64 || c->wm_pred_hidden > 1024 ||
        c->wm_proj_hidden < 64 || c->wm_proj_hidden % 64 || c->wm_proj_hidden > 16384 || c->wm_action_dim < 1 ||
        c->wm_action_dim > 64 || c->wm_window < 1 || c->wm_window > 32 || !c->has_cls)
      return JEPA_B200_ERR_SHAPE;
  }
  if (c->rope && (c->has_cls || c->frames / c->tubelet > kRopeMaxPos || c->img_h / c->patch > kRopeMaxPos ||
                  c->img_w / c->patch > kRopeMaxPos))
    return JEPA_B200_ERR_SHAPE;
  return JEPA_B200_OK;
}

int alloc_ws(jepa_b200_model* m, void** p, size_t bytes) {
  if (cudaMalloc(p, bytes) != cudaSuccess) return JEPA_B200_ERR_CUDA;
  m->ws_allocs.push_back(*p);
  return JEPA_B200_OK;
}

int prepare_block_ops(jepa_b200_model* m, const LayerW& L, BlockOps& ops, float* Xres, int R, bool rope) {
  const int D = m->cfg.dim, Mh = m->cfg.mlp;
  QkvDst qd;
  if (rope) {  // the encoder blocks of a rotary model
    qd.rope = m->rope;
    qd.rope_ppf = (m->cfg.img_h / m->cfg.patch) * (m->cfg.img_w / m->cfg.patch);
    qd.rope_pw = m->cfg.img_w / m->cfg.patch;
  }
  qd.q = m->Q;
  qd.k = m->Kb;
  qd.vt = m->Vt;
  qd.ntok = m->N;
  qd.heads = m->cfg.heads;
  qd.npad = m->npad;
  qd.first_part = 0;
  qd.dim = D;
  int s;
  if ((s = gemm_prepare(&ops.qkv, m->Y, R, D, L.qkv, L.b_qkv, EPI_QKV, m->Q, 3 * D, &qd, nullptr))) return s;
  if ((s = gemm_prepare(&ops.out, m->O, R, D, L.out, L.b_out, EPI_RESID_F32, Xres, D, nullptr, nullptr))) return s;
  if ((s = gemm_prepare(&ops.up, m->Y, R, D, L.up, L.b_up, EPI_GELU_F16, m->H, Mh, nullptr, nullptr))) return s;
  if ((s = gemm_prepare(&ops.down, m->H, R, Mh, L.down, L.b_down, EPI_RESID_F32, Xres, D, nullptr, nullptr)))
    return s;
  return JEPA_B200_OK;
}

// Workspace buffers for B clips; every launch's parameters (row counts,
// tensor maps) for B clips.
int alloc_workspace(jepa_b200_model* m, int B);
int prepare_ops(jepa_b200_model* m, int B);

// Workspace for at least B clips (grown, never shrunk) and the ops for
// exactly B clips (rebuilt whenever B changes).
int ensure_workspace(jepa_b200_model* m, int B) {
  int s = JEPA_B200_OK;
  if (B > m->ws_B) {
    cudaDeviceSynchronize();
    if (m->graph) {  // it points into the workspace about to be freed
      cudaGraphExecDestroy(m->graph);
      m->graph = nullptr;
    }
    m->g_key = EncodeKey();
    free_list(m->ws_allocs);
    m->ws_B = 0;
    m->ops_B = 0;
    if ((s = alloc_workspace(m, B))) return s;
    m->ws_B = B;
  }
  if (B != m->ops_B) {
    m->ops_B = 0;
    if ((s = prepare_ops(m, B))) return s;
    m->ops_B = B;
  }
  return JEPA_B200_OK;
}

int alloc_workspace(jepa_b200_model* m, int B) {
  const jepa_b200_config& c = m->cfg;
  const size_t R = static_cast<size_t>(B) * m->N;
  const size_t D = c.dim;
  int s = JEPA_B200_OK;
  s = s ? s : alloc_ws(m, reinterpret_cast<void**>(&m->X), R * D * 4);
  s = s ? s : alloc_ws(m, reinterpret_cast<void**>(&m->Y), R * D * 2);
  s = s ? s : alloc_ws(m, reinterpret_cast<void**>(&m->Q), R * D * 2);
  s = s ? s : alloc_ws(m, reinterpret_cast<void**>(&m->Kb), R * D * 2);
  const size_t vt_bytes = static_cast<size_t>(B) * c.heads * 64 * m->npad * 2;
  s = s ? s : alloc_ws(m, reinterpret_cast<void**>(&m->Vt), vt_bytes);
  s = s ? s : alloc_ws(m, reinterpret_cast<void**>(&m->O), R * D * 2);
  s = s ? s : alloc_ws(m, reinterpret_cast<void**>(&m->H), R * c.mlp * 2);
  s = s ? s : alloc_ws(m, reinterpret_cast<void**>(&m->Yf), R * D * 4);
  s = s ? s : alloc_ws(m, reinterpret_cast<void**>(&m->partial), static_cast<size_t>(mean_pool_partial_floats(B, c.dim)) * 4);
  s = s ? s : alloc_ws(m, reinterpret_cast<void**>(&m->hq), D * 4);
  s = s ? s : alloc_ws(m, reinterpret_cast<void**>(&m->hattn), B * D * 4);
  s = s ? s : alloc_ws(m, reinterpret_cast<void**>(&m->hz), B * D * 4);
  s = s ? s : alloc_ws(m, reinterpret_cast<void**>(&m->hzn), B * D * 4);
  s = s ? s : alloc_ws(m, reinterpret_cast<void**>(&m->hu), static_cast<size_t>(B) * c.mlp * 4);
  s = s ? s : alloc_ws(m, reinterpret_cast<void**>(&m->Ape), static_cast<size_t>(B) * m->Np * m->Kpe_pad * 2);
  if (c.wm_depth > 0)
    s = s ? s : alloc_ws(m, reinterpret_cast<void**>(&m->hp), static_cast<size_t>(B) * c.wm_proj_hidden * 4);
  if (s) {
    free_list(m->ws_allocs);
    return s;
  }
  // V^T columns past the last token stay zero: the attention multiplies them by p = 0
  if (cudaMemset(m->Vt, 0, vt_bytes) != cudaSuccess) return JEPA_B200_ERR_CUDA;
  return JEPA_B200_OK;
}

int prepare_ops(jepa_b200_model* m, int B) {
  const jepa_b200_config& c = m->cfg;
  const size_t R = static_cast<size_t>(B) * m->N;
  int s = JEPA_B200_OK;
  const int Ri = static_cast<int>(R);
  m->enc_ops.assign(m->enc.size(), BlockOps());
  for (size_t l = 0; l < m->enc.size(); ++l)
    if ((s = prepare_block_ops(m, m->enc[l], m->enc_ops[l], m->X, Ri, m->cfg.rope != 0))) return s;
  m->head_ops.assign(m->head.size(), BlockOps());
  for (size_t l = 0; l < m->head.size(); ++l)
    if ((s = prepare_block_ops(m, m->head[l], m->head_ops[l], m->Yf, Ri, false))) return s;
  PatchSrc ps;
  ps.pixels = nullptr;
  ps.T = c.frames;
  ps.H = c.img_h;
  ps.W = c.img_w;
  ps.patch = c.patch;
  ps.tubelet = c.tubelet;
  ps.n_patches = m->Np;
  ps.k_real = m->Kpe;
  ps.pos = m->pos;
  ps.ntok = m->N;
  ps.has_cls = c.has_cls ? 1 : 0;
  // patch-embed: the unfolded patch matrix (launch_patchify) through the
  // TMA-fed GEMM, whose epilogue adds the bias and positional row in place
  if ((s = gemm_prepare(&m->pe_op, m->Ape, B * m->Np, m->Kpe_pad, m->pe, m->b_pe, EPI_PATCH, m->X, c.dim, nullptr,
                        &ps)))
    return s;
  if ((s = attn_prepare(&m->attn_enc, m->Q, m->Kb, m->Vt, B, c.heads, m->N, m->npad, c.mask, c.has_cls, m->ppf,
                        m->O)))
    return s;
  if ((s = attn_prepare(&m->attn_head, m->Q, m->Kb, m->Vt, B, c.heads, m->N, m->npad, JEPA_B200_MASK_BIDIR, 0, 1,
                        m->O)))
    return s;
  m->attn_enc.bf16 = m->attn_head.bf16 = c.act_bf16 != 0;
  if (m->has_head) {
    QkvDst qd;
    qd.q = nullptr;
    qd.k = m->Kb;
    qd.vt = m->Vt;
    qd.ntok = m->N;
    qd.heads = c.heads;
    qd.npad = m->npad;
    qd.first_part = 1;
    qd.dim = c.dim;
    if ((s = gemm_prepare(&m->kv_op, m->Y, Ri, c.dim, m->xkv, m->b_xkv, EPI_QKV, m->Kb, 2 * c.dim, &qd, nullptr)))
      return s;
  }
  return JEPA_B200_OK;
}

// The kernel sequence of one forward on `st` (workspace and ops ready).
int enqueue_forward(jepa_b200_model* m, const float* pixels, int B, int pool, float* out, cudaStream_t st);

// Capture the forward into m->graph (replacing the previous one).
int capture_forward(jepa_b200_model* m, const EncodeKey& key) {
  if (m->graph) {
    cudaGraphExecDestroy(m->graph);
    m->graph = nullptr;
  }
  if (!m->cap_stream && cudaStreamCreateWithFlags(&m->cap_stream, cudaStreamNonBlocking) != cudaSuccess)
    return JEPA_B200_ERR_CUDA;
  if (cudaStreamBeginCapture(m->cap_stream, cudaStreamCaptureModeThreadLocal) != cudaSuccess)
    return JEPA_B200_ERR_CUDA;
  m->launches = 0;
  const int s = enqueue_forward(m, key.pixels, key.B, key.pool, const_cast<float*>(key.out), m->cap_stream);
  cudaGraph_t g = nullptr;
  const cudaError_t e = cudaStreamEndCapture(m->cap_stream, &g);
  if (s || e != cudaSuccess) {
    if (g) cudaGraphDestroy(g);
    cudaGetLastError();
    return s ? s : JEPA_B200_ERR_CUDA;
  }
  const cudaError_t ei = cudaGraphInstantiate(&m->graph, g, 0);
  cudaGraphDestroy(g);
  if (ei != cudaSuccess) {
    m->graph = nullptr;
    return JEPA_B200_ERR_CUDA;
  }
  m->g_key = key;
  m->g_launches = m->launches;
  return JEPA_B200_OK;
}

// Event pair around one launch while profiling is on.
size_t prof_event(jepa_b200_model* m) {
  if (m->prof_used == m->prof_events.size()) {
    cudaEvent_t e = nullptr;
    if (cudaEventCreate(&e) != cudaSuccess) return SIZE_MAX;
    m->prof_events.push_back(e);
  }
  return m->prof_used++;
}

struct ProfScope {
  jepa_b200_model* m;
  int cls;
  cudaStream_t st;
  size_t e0 = SIZE_MAX;
  ProfScope(jepa_b200_model* m_, int cls_, cudaStream_t st_) : m(m_), cls(cls_), st(st_) {
    if (m->prof) {
      e0 = prof_event(m);
      if (e0 != SIZE_MAX) cudaEventRecord(m->prof_events[e0], st);
    }
  }
  ~ProfScope() {
    if (m->prof && e0 != SIZE_MAX) {
      const size_t e1 = prof_event(m);
      if (e1 != SIZE_MAX) {
        cudaEventRecord(m->prof_events[e1], st);
        m->prof_recs.push_back({cls, e0, e1});
      }
    }
  }
};

#define JB_TRY(expr)            \
  do {                          \
    const int _s = (expr);      \
    if (_s != JEPA_B200_OK) return _s; \
  } while (0)

// One pre-LN block on the residual Xres [R, D] (D: the encoder's width, or
// the predictor's with its own LN output buffer Y).
int run_block(jepa_b200_model* m, const LayerW& L, const BlockOps& ops, const AttnOp& at, float* Xres, int R,
              cudaStream_t st, int D = 0, __half* Y = nullptr) {
  if (!D) D = m->cfg.dim;
  if (!Y) Y = m->Y;
  const float eps = m->cfg.ln_eps;
  {
    ProfScope ps(m, JEPA_B200_KC_LAYERNORM, st);
    JB_TRY(launch_layernorm(Xres, R, D, 1, L.ln1_g, L.ln1_b, eps, Y, true, st, m->cfg.act_bf16 != 0));
  }
  {
    ProfScope ps(m, JEPA_B200_KC_GEMM_QKV, st);
    JB_TRY(gemm_launch(ops.qkv, st, m->err, m->timeout_ns));
  }
  {
    ProfScope ps(m, JEPA_B200_KC_ATTENTION, st);
    JB_TRY(attn_launch(at, st, m->err, m->timeout_ns));
  }
  {
    ProfScope ps(m, JEPA_B200_KC_GEMM_OUT, st);
    JB_TRY(gemm_launch(ops.out, st, m->err, m->timeout_ns));
  }
  {
    ProfScope ps(m, JEPA_B200_KC_LAYERNORM, st);
    JB_TRY(launch_layernorm(Xres, R, D, 1, L.ln2_g, L.ln2_b, eps, Y, true, st, m->cfg.act_bf16 != 0));
  }
  {
    ProfScope ps(m, JEPA_B200_KC_GEMM_UP, st);
    JB_TRY(gemm_launch(ops.up, st, m->err, m->timeout_ns));
  }
  {
    ProfScope ps(m, JEPA_B200_KC_GEMM_DOWN, st);
    JB_TRY(gemm_launch(ops.down, st, m->err, m->timeout_ns));
  }
  m->launches += 7;
  return JEPA_B200_OK;
}

int run_embed_and_blocks(jepa_b200_model* m, const float* pixels, int B, int n_layers, cudaStream_t st) {
  const jepa_b200_config& c = m->cfg;
  const int R = B * m->N;
  {
    ProfScope ps(m, JEPA_B200_KC_PATCH_EMBED, st);
    PatchSrc src = m->pe_op.p.patch;
    JB_TRY(launch_patchify(pixels, src, B, m->Kpe_pad, m->Ape, st, c.act_bf16 != 0));
    JB_TRY(gemm_launch(m->pe_op, st, m->err, m->timeout_ns));
    m->launches += 2;
    if (c.has_cls) {
      JB_TRY(launch_cls_rows(m->X, B, m->N, c.dim, m->cls, m->pos, st));
      m->launches += 1;
    }
  }
  for (int l = 0; l < n_layers; ++l) JB_TRY(run_block(m, m->enc[l], m->enc_ops[l], m->attn_enc, m->X, R, st));
  return JEPA_B200_OK;
}

int run_head(jepa_b200_model* m, int B, float* out, cudaStream_t st) {
  const jepa_b200_config& c = m->cfg;
  const int R = B * m->N, D = c.dim;
  const float eps = c.ln_eps;
  for (size_t l = 0; l < m->head.size(); ++l)
    JB_TRY(run_block(m, m->head[l], m->head_ops[l], m->attn_head, m->Yf, R, st));
  ProfScope ps(m, JEPA_B200_KC_POOL_HEAD, st);
  JB_TRY(launch_layernorm(m->Yf, R, D, 1, m->lnkv_g, m->lnkv_b, eps, m->Y, true, st, c.act_bf16 != 0));
  JB_TRY(gemm_launch(m->kv_op, st, m->err, m->timeout_ns));
  // q = W_q query + b_q (the learned query, shared by every clip)
  JB_TRY(launch_gemv(m->query, 1, D, m->xq, m->b_xq, 0, nullptr, 0, m->hq, st));
  JB_TRY(launch_xattn_1q(m->hq, m->Kb, m->Vt, B, c.heads, m->N, m->npad, m->hattn, st, c.act_bf16 != 0));
  // z = query + W_out attn + b_out
  JB_TRY(launch_gemv(m->hattn, B, D, m->xout, m->b_xout, 2, m->query, 0, m->hz, st));
  JB_TRY(launch_layernorm(m->hz, B, D, 1, m->ln2x_g, m->ln2x_b, eps, m->hzn, false, st));
  JB_TRY(launch_gemv(m->hzn, B, D, m->xup, m->b_xup, 1, nullptr, 0, m->hu, st));
  JB_TRY(launch_gemv(m->hu, B, c.mlp, m->xdown, m->b_xdown, 2, m->hz, D, m->hz, st));
  JB_TRY(launch_gemv(m->hz, B, D, m->hcls, m->b_cls, 0, nullptr, 0, out, st));
  m->launches += 9;
  return JEPA_B200_OK;
}

size_t out_elems(const jepa_b200_model* m, int B, int pool) {
  switch (pool) {
    case JEPA_B200_POOL_NONE: return static_cast<size_t>(B) * m->N * m->cfg.dim;
    case JEPA_B200_POOL_MEAN:
    case JEPA_B200_POOL_CLS:
    case JEPA_B200_POOL_LEWM: return static_cast<size_t>(B) * m->cfg.dim;
    case JEPA_B200_POOL_ATTENTIVE: return static_cast<size_t>(B) * m->cfg.n_classes;
    default: return 0;
  }
}

int check_encode_args(jepa_b200_model* m, const void* pixels, int B, int pool, const void* out, size_t out_bytes) {
  if (!m || !pixels || !out || B < 1) return JEPA_B200_ERR_ARG;
  if (pool < JEPA_B200_POOL_NONE || pool > JEPA_B200_POOL_LEWM) return JEPA_B200_ERR_ARG;
  if (pool == JEPA_B200_POOL_LEWM && m->cfg.wm_depth < 1) return JEPA_B200_ERR_MISSING_TENSOR;
  if (pool == JEPA_B200_POOL_ATTENTIVE && !m->has_head) return JEPA_B200_ERR_MISSING_TENSOR;
  if (pool == JEPA_B200_POOL_CLS && !m->cfg.has_cls) return JEPA_B200_ERR_ARG;
  if (static_cast<long long>(B) * m->N > (1ll << 31) / 4096) return JEPA_B200_ERR_SHAPE;
  if (out_bytes < out_elems(m, B, pool) * 4) return JEPA_B200_ERR_SHAPE;
  if ((reinterpret_cast<uintptr_t>(pixels) & 15) || (reinterpret_cast<uintptr_t>(out) & 15)) return JEPA_B200_ERR_ARG;
  return JEPA_B200_OK;
}

int enqueue_forward(jepa_b200_model* m, const float* pixels, int B, int pool, float* out, cudaStream_t st) {
  const jepa_b200_config& c = m->cfg;
  const int R = B * m->N, D = c.dim;
  int s = run_embed_and_blocks(m, pixels, B, c.depth, st);
  if (s) return s;
  {
    ProfScope ps(m, JEPA_B200_KC_LAYERNORM, st);
    if (pool == JEPA_B200_POOL_NONE)
      s = launch_layernorm(m->X, R, D, 1, m->norm_g, m->norm_b, c.ln_eps, out, false, st);
    else if (pool == JEPA_B200_POOL_CLS)
      s = launch_layernorm(m->X, B, D, m->N, m->norm_g, m->norm_b, c.ln_eps, out, false, st);
    else if (pool == JEPA_B200_POOL_LEWM)
      s = launch_layernorm(m->X, B, D, m->N, m->norm_g, m->norm_b, c.ln_eps, m->hz, false, st);
    else
      s = launch_layernorm(m->X, R, D, 1, m->norm_g, m->norm_b, c.ln_eps, m->Yf, false, st);
    m->launches += 1;
  }
  if (!s && pool == JEPA_B200_POOL_MEAN) {
    ProfScope ps(m, JEPA_B200_KC_POOL_HEAD, st);
    s = launch_mean_pool(m->Yf, B, m->N, D, c.has_cls ? 1 : 0, m->partial, out, st);
    m->launches += 2;
  }
  if (!s && pool == JEPA_B200_POOL_ATTENTIVE) s = run_head(m, B, out, st);
  if (!s && pool == JEPA_B200_POOL_LEWM) {  // the LeWM projector on the final-normed CLS rows
    ProfScope ps(m, JEPA_B200_KC_POOL_HEAD, st);
    s = launch_gemv(m->hz, B, D, m->wproj0, m->b_wproj0, 1, nullptr, 0, m->hp, st);
    if (!s) s = launch_gemv(m->hp, B, c.wm_proj_hidden, m->wproj2, m->b_wproj2, 0, nullptr, 0, out, st);
    m->launches += 2;
  }
  return s;
}

// ------------------------------------------------------------ predictor --
// Workspace for `rows` sequence rows (B * (n_ctx + n_tgt)), `crows` context
// rows and `trows` target rows, grown and never shrunk; every buffer whose
// 64-dim head rows the QKV epilogue fills only partly (32-dim heads) starts
// zeroed, so the dims it never writes stay zero.
int pred_workspace(jepa_b200_model* m, size_t rows, size_t crows, size_t trows, size_t vt_elems) {
  if (rows <= m->pws_rows && crows <= m->pws_ctx_rows && trows <= m->pws_tgt_rows && vt_elems <= m->pws_vt)
    return JEPA_B200_OK;
  rows = std::max(rows, m->pws_rows);
  crows = std::max(crows, m->pws_ctx_rows);
  trows = std::max(trows, m->pws_tgt_rows);
  const size_t vt_cap = std::max(vt_elems, m->pws_vt);
  cudaDeviceSynchronize();
  free_list(m->pws_allocs);
  m->pws_rows = m->pws_ctx_rows = m->pws_tgt_rows = m->pws_vt = 0;
  m->pops_B = 0;
  const jepa_b200_config& c = m->cfg;
  const size_t Dp = c.pred_dim, Mp = c.pred_mlp, D = c.dim;
  // Q, K: [B*h, L, 64] = rows * h * 64 halves; V^T: [B*h, 64, Lpad] (vt_cap)
  const size_t qk_elems = rows * c.pred_heads * 64;
  auto get = [&](void** p, size_t bytes, bool zero) -> int {
    if (cudaMalloc(p, bytes) != cudaSuccess) return JEPA_B200_ERR_CUDA;
    m->pws_allocs.push_back(*p);
    if (zero && cudaMemset(*p, 0, bytes) != cudaSuccess) return JEPA_B200_ERR_CUDA;
    return JEPA_B200_OK;
  };
  int s = JEPA_B200_OK;
  s = s ? s : get(reinterpret_cast<void**>(&m->pX), rows * Dp * 4, false);
  s = s ? s : get(reinterpret_cast<void**>(&m->pY), rows * Dp * 2, false);
  s = s ? s : get(reinterpret_cast<void**>(&m->pQ), qk_elems * 2, true);
  s = s ? s : get(reinterpret_cast<void**>(&m->pK), qk_elems * 2, true);
  s = s ? s : get(reinterpret_cast<void**>(&m->pVt), vt_cap * 2, true);
  s = s ? s : get(reinterpret_cast<void**>(&m->pO), rows * Dp * 2, false);
  s = s ? s : get(reinterpret_cast<void**>(&m->pH), rows * Mp * 2, false);
  s = s ? s : get(reinterpret_cast<void**>(&m->pA), crows * D * 2, false);
  s = s ? s : get(reinterpret_cast<void**>(&m->pE), crows * Dp * 4, false);
  s = s ? s : get(reinterpret_cast<void**>(&m->pT), trows * Dp * 2, false);
  s = s ? s : get(reinterpret_cast<void**>(&m->pidx), static_cast<size_t>(2) * m->N * sizeof(int), false);
  if (s) {
    free_list(m->pws_allocs);
    return s;
  }
  m->pws_rows = rows;
  m->pws_ctx_rows = crows;
  m->pws_tgt_rows = trows;
  m->pws_vt = vt_cap;
  m->pidx_host.clear();
  return JEPA_B200_OK;
}

int prepare_pred_ops(jepa_b200_model* m, const float* tokens, int B, int nc, int nt, float* out) {
  const jepa_b200_config& c = m->cfg;
  const int Dp = c.pred_dim, Mp = c.pred_mlp, L = nc + nt, R = B * L;
  const int hd = Dp / c.pred_heads, Lpad = (L + 127) / 128 * 128;
  int s;
  // context rows: tokens (gathered, f16) -> pred.embed -> pE f32
  if ((s = gemm_prepare(&m->pembed_op, m->pA, B * nc, c.dim, m->pembed, m->b_pembed, EPI_F32, m->pE, Dp, nullptr,
                        nullptr)))
    return s;
  m->pred_ops.assign(m->pred.size(), BlockOps());
  for (size_t l = 0; l < m->pred.size(); ++l) {
    const LayerW& W = m->pred[l];
    BlockOps& ops = m->pred_ops[l];
    QkvDst qd;
    qd.q = m->pQ;
    qd.k = m->pK;
    qd.vt = m->pVt;
    qd.ntok = L;
    qd.heads = c.pred_heads;
    qd.npad = Lpad;
    qd.dim = Dp;
    qd.head_dim = hd;
    if ((s = gemm_prepare(&ops.qkv, m->pY, R, Dp, W.qkv, W.b_qkv, EPI_QKV, m->pQ, 3 * Dp, &qd, nullptr))) return s;
    if ((s = gemm_prepare(&ops.out, m->pO, R, Dp, W.out, W.b_out, EPI_RESID_F32, m->pX, Dp, nullptr, nullptr)))
      return s;
    if ((s = gemm_prepare(&ops.up, m->pY, R, Dp, W.up, W.b_up, EPI_GELU_F16, m->pH, Mp, nullptr, nullptr))) return s;
    if ((s = gemm_prepare(&ops.down, m->pH, R, Mp, W.down, W.b_down, EPI_RESID_F32, m->pX, Dp, nullptr, nullptr)))
      return s;
  }
  if ((s = attn_prepare(&m->pattn, m->pQ, m->pK, m->pVt, B, c.pred_heads, L, Lpad, JEPA_B200_MASK_BIDIR, 0, 1, m->pO,
                        hd)))
    return s;
  m->pattn.bf16 = c.act_bf16 != 0;
  // target rows: pred.norm -> pT f16 -> pred.proj -> out f32 [B * nt, dim]
  if ((s = gemm_prepare(&m->pproj_op, m->pT, B * nt, Dp, m->pproj, m->b_pproj, EPI_F32, out, c.dim, nullptr,
                        nullptr)))
    return s;
  return JEPA_B200_OK;
}

int enqueue_predict(jepa_b200_model* m, const float* tokens, int B, int nc, int nt, cudaStream_t st) {
  const jepa_b200_config& c = m->cfg;
  const int Dp = c.pred_dim, L = nc + nt, R = B * L;
  const int* ctx = m->pidx;
  const int* tgt = m->pidx + m->N;
  {
    ProfScope ps(m, JEPA_B200_KC_PATCH_EMBED, st);
    JB_TRY(launch_gather_rows_f16(tokens, ctx, B, m->N, nc, c.dim, m->pA, st, c.act_bf16 != 0));
    JB_TRY(gemm_launch(m->pembed_op, st, m->err, m->timeout_ns));
    JB_TRY(launch_pred_assemble(m->pE, m->pmask, m->ppos, ctx, tgt, B, nc, nt, Dp, m->pX, st));
  }
  m->launches += 3;
  for (size_t l = 0; l < m->pred.size(); ++l)
    JB_TRY(run_block(m, m->pred[l], m->pred_ops[l], m->pattn, m->pX, R, st, Dp, m->pY));
  {
    ProfScope ps(m, JEPA_B200_KC_POOL_HEAD, st);
    JB_TRY(launch_layernorm_rows(m->pX, B * nt, Dp, nt, L, nc, m->pnorm_g, m->pnorm_b, c.ln_eps, m->pT, true, st,
                                 c.act_bf16 != 0));
    JB_TRY(gemm_launch(m->pproj_op, st, m->err, m->timeout_ns));
  }
  m->launches += 2;
  return JEPA_B200_OK;
}

}  // namespace

static void load_sequence(Loader& L);
static void load_world_model(Loader& L);

extern "C" {

const char* jepa_b200_status_str(int s) {
  switch (s) {
    case JEPA_B200_OK: return "ok";
    case JEPA_B200_ERR_ARG: return "invalid argument";
    case JEPA_B200_ERR_MISSING_TENSOR: return "missing tensor";
    case JEPA_B200_ERR_SHAPE: return "wrong shape or size";
    case JEPA_B200_ERR_DTYPE: return "dtype not allowed for this tensor";
    case JEPA_B200_ERR_CUDA: return "CUDA call failed";
    case JEPA_B200_ERR_TIMEOUT: return "a bounded device-side wait ran out";
    case JEPA_B200_ERR_UNSUPPORTED: return "not supported";
    default: return "unknown status";
  }
}

int jepa_b200_load_weights(const jepa_b200_config* cfg, const jepa_b200_tensor* table, int n_tensors, int device,
                           jepa_b200_model** out_model) {
  if (!out_model) return JEPA_B200_ERR_ARG;
  *out_model = nullptr;
  int s = validate_config(cfg);
  if (s) return s;
  if (!table || n_tensors < 1) return JEPA_B200_ERR_ARG;
  if (device < 0) return JEPA_B200_ERR_ARG;
  jepa_b200_model* m = new jepa_b200_model();
  m->cfg = *cfg;
  m->device = device;
  const jepa_b200_config& c = *cfg;
  m->ppf = (c.img_h / c.patch) * (c.img_w / c.patch);
  m->Np = (c.frames / c.tubelet) * m->ppf;
  m->N = m->Np + (c.has_cls ? 1 : 0);
  m->npad = (m->N + 127) / 128 * 128;
  m->Kpe = 3 * c.tubelet * c.patch * c.patch;
  m->Kpe_pad = (m->Kpe + 63) / 64 * 64;
  m->has_head = c.n_classes > 0;

  for (int i = 0; i < n_tensors; ++i)
    if (!table[i].name) {
      delete m;
      return JEPA_B200_ERR_ARG;
    }
  // pass 1 validates the whole table on the host; pass 2 converts and uploads
  {
    jepa_b200_model probe;
    probe.cfg = m->cfg;
    probe.N = m->N;
    probe.Np = m->Np;
    probe.Kpe = m->Kpe;
    probe.Kpe_pad = m->Kpe_pad;
    probe.has_head = m->has_head;
    Loader V;
    V.m = &probe;
    V.dry = true;
    for (int i = 0; i < n_tensors; ++i)
      if (!V.tab.emplace(table[i].name, &table[i]).second) {  // a name given twice
        delete m;
        return JEPA_B200_ERR_ARG;
      }
    load_sequence(V);
    if (V.status != JEPA_B200_OK) {
      delete m;
      return V.status;
    }
  }
  int ndev = 0;
  if (cudaGetDeviceCount(&ndev) != cudaSuccess || device < 0 || device >= ndev) {
    delete m;
    return JEPA_B200_ERR_CUDA;
  }
  DeviceGuard guard(device);
  Loader L;
  L.m = m;
  for (int i = 0; i < n_tensors; ++i) L.tab[table[i].name] = &table[i];
  load_sequence(L);
  if (L.status == JEPA_B200_OK && cudaDeviceSynchronize() != cudaSuccess) L.status = JEPA_B200_ERR_CUDA;
  if (L.status == JEPA_B200_OK) {
    if (cudaMalloc(&m->err, sizeof(DevErr)) != cudaSuccess || cudaMemset(m->err, 0, sizeof(DevErr)) != cudaSuccess ||
        cudaEventCreate(&m->ev0) != cudaSuccess || cudaEventCreate(&m->ev1) != cudaSuccess)
      L.status = JEPA_B200_ERR_CUDA;
  }
  if (L.status != JEPA_B200_OK) {
    jepa_b200_free(m);
    return L.status;
  }
  *out_model = m;
  return JEPA_B200_OK;
}

}  // extern "C"

static void load_sequence(Loader& L) {
  jepa_b200_model* m = L.m;
  const jepa_b200_config& c = m->cfg;
  const int64_t D = c.dim, Mh = c.mlp;
  {
    const jepa_b200_tensor* t = L.get("enc.patch_embed.weight", {D, 3, c.tubelet, c.patch, c.patch});
    if (t && t->dtype != JEPA_B200_F32 && t->dtype != JEPA_B200_F16) L.status = JEPA_B200_ERR_DTYPE;
    if (t && L.status == JEPA_B200_OK) m->pe = L.matrix({t}, m->Kpe, m->Kpe_pad);
  }
  m->b_pe = L.vec("enc.patch_embed.bias", D);
  if (c.rope) {
    // (cos, sin) of pos * 10000^(-2i/20) for every axis position and pair i,
    // in double precision, rounded once to f32
    std::vector<float2> tab(static_cast<size_t>(3) * kRopeMaxPos * 10);
    for (int a = 0; a < 3; ++a)
      for (int pos = 0; pos < kRopeMaxPos; ++pos)
        for (int i = 0; i < 10; ++i) {
          const double th = pos * std::pow(10000.0, -2.0 * i / 20.0);
          tab[(static_cast<size_t>(a) * kRopeMaxPos + pos) * 10 + i] =
              make_float2(static_cast<float>(std::cos(th)), static_cast<float>(std::sin(th)));
        }
    m->rope = static_cast<float2*>(L.dalloc(tab.size() * sizeof(float2)));
    if (m->rope) L.upload(m->rope, tab.data(), tab.size() * sizeof(float2));
  } else {
    m->pos = L.table2d("enc.pos_embed", m->N, D);
  }
  if (c.has_cls) m->cls = L.vec("enc.cls_token", D);
  m->enc.resize(c.depth);
  for (int l = 0; l < c.depth; ++l) L.block(m->enc[l], "enc.blk." + std::to_string(l) + ".", D, Mh);
  m->norm_g = L.vec("enc.norm.weight", D);
  m->norm_b = L.vec("enc.norm.bias", D);
  if (m->has_head) {
    m->head.resize(c.head_sa_blocks);
    for (int l = 0; l < c.head_sa_blocks; ++l) L.block(m->head[l], "head.blk." + std::to_string(l) + ".", D, Mh);
    m->query = L.vec("head.query", D);
    m->lnkv_g = L.vec("head.ln_kv.weight", D);
    m->lnkv_b = L.vec("head.ln_kv.bias", D);
    m->xq = L.mat("head.xattn.q.weight", D, D);
    m->b_xq = L.vec("head.xattn.q.bias", D);
    {
      const jepa_b200_tensor* tk = L.get("head.xattn.k.weight", {D, D});
      const jepa_b200_tensor* tv = L.get("head.xattn.v.weight", {D, D});
      if (tk && tv) m->xkv = L.matrix({tk, tv}, D, D);
      const jepa_b200_tensor* bk = L.get("head.xattn.k.bias", {D});
      const jepa_b200_tensor* bv = L.get("head.xattn.v.bias", {D});
      if (bk && bv) {
        std::vector<float> v = L.host_floats(bk), w = L.host_floats(bv);
        v.insert(v.end(), w.begin(), w.end());
        m->b_xkv = static_cast<float*>(L.dalloc(v.size() * 4));
        if (m->b_xkv) L.upload(m->b_xkv, v.data(), v.size() * 4);
      }
    }
    m->xout = L.mat("head.xattn.out.weight", D, D);
    m->b_xout = L.vec("head.xattn.out.bias", D);
    m->ln2x_g = L.vec("head.xattn.ln2.weight", D);
    m->ln2x_b = L.vec("head.xattn.ln2.bias", D);
    m->xup = L.mat("head.xattn.ffn_up.weight", Mh, D);
    m->b_xup = L.vec("head.xattn.ffn_up.bias", Mh);
    m->xdown = L.mat("head.xattn.ffn_down.weight", D, Mh);
    m->b_xdown = L.vec("head.xattn.ffn_down.bias", D);
    m->hcls = L.mat("head.cls.weight", c.n_classes, D);
    m->b_cls = L.vec("head.cls.bias", c.n_classes);
  }
  if (c.pred_depth > 0) {
    const int64_t Dp = c.pred_dim, Mp = c.pred_mlp;
    m->pembed = L.mat("pred.embed.weight", Dp, D);
    m->b_pembed = L.vec("pred.embed.bias", Dp);
    m->pmask = L.table2d("pred.mask_tokens", 1, Dp);
    m->ppos = L.table2d("pred.pos_embed", m->N, Dp);
    m->pred.resize(c.pred_depth);
    for (int l = 0; l < c.pred_depth; ++l) L.block(m->pred[l], "pred.blk." + std::to_string(l) + ".", Dp, Mp);
    m->pnorm_g = L.vec("pred.norm.weight", Dp);
    m->pnorm_b = L.vec("pred.norm.bias", Dp);
    m->pproj = L.mat("pred.proj.weight", D, Dp);
    m->b_pproj = L.vec("pred.proj.bias", D);
  }
  if (c.wm_depth > 0) load_world_model(L);
}

// The LeWM world model: the projector as two matrices for the few-row
// kernels, the predictor's matrices in three 16-bit arenas (row layout in
// WmArena), its vectors in f32.
static void load_world_model(Loader& L) {
  jepa_b200_model* m = L.m;
  const jepa_b200_config& c = m->cfg;
  const int64_t D = c.dim, Mh = c.wm_mlp, Hq = c.wm_pred_hidden, Hp = c.wm_proj_hidden, A = c.wm_action_dim;
  const int depth = c.wm_depth;
  m->wproj0 = L.mat("enc.proj.0.weight", Hp, D);
  m->b_wproj0 = L.vec("enc.proj.0.bias", Hp);
  m->wproj2 = L.mat("enc.proj.2.weight", D, Hp);
  m->b_wproj2 = L.vec("enc.proj.2.bias", D);
  WmArena& a = m->wm;
  a.D = static_cast<int>(D);
  a.mlp = static_cast<int>(Mh);
  a.hq = static_cast<int>(Hq);
  a.bf16 = c.act_bf16 ? 1 : 0;
  const int64_t blk = 10 * D + Mh;
  a.rows_d = static_cast<int>(D + depth * blk + Hq);
  a.rows_m = static_cast<int>(depth * D);
  a.rows_h = static_cast<int>(D);
  a.d = L.dalloc(static_cast<size_t>(a.rows_d) * D * 2);
  a.m = L.dalloc(static_cast<size_t>(a.rows_m) * Mh * 2);
  a.h = L.dalloc(static_cast<size_t>(a.rows_h) * Hq * 2);
  L.arena_put(a.d, 0, "pred.action_embed.2.weight", D, D);
  for (int b = 0; b < depth; ++b) {
    const std::string p = "pred.blk." + std::to_string(b) + ".";
    const int64_t base = D + b * blk;
    L.arena_put(a.d, base, p + "adaln.weight", 6 * D, D);
    L.arena_put(a.d, base + 6 * D, p + "attn_qkv.weight", 3 * D, D);
    L.arena_put(a.d, base + 9 * D, p + "attn_out.weight", D, D);
    L.arena_put(a.d, base + 10 * D, p + "ffn_up.weight", Mh, D);
    L.arena_put(a.m, b * D, p + "ffn_down.weight", D, Mh);
  }
  L.arena_put(a.d, D + depth * blk, "pred.proj.0.weight", Hq, D);
  L.arena_put(a.h, 0, "pred.proj.2.weight", D, Hq);
  m->wm_w_act0 = L.table2d("pred.action_embed.0.weight", D, A);
  m->wm_b_act0 = L.vec("pred.action_embed.0.bias", D);
  m->wm_b_act2 = L.vec("pred.action_embed.2.bias", D);
  m->wm_pos = L.table2d("pred.pos_embed", c.wm_window, D);
  m->wm_b_ada = L.vec_stack("pred.blk.", "adaln.bias", depth, 6 * D);
  m->wm_b_qkv = L.vec_stack("pred.blk.", "attn_qkv.bias", depth, 3 * D);
  m->wm_b_out = L.vec_stack("pred.blk.", "attn_out.bias", depth, D);
  m->wm_b_up = L.vec_stack("pred.blk.", "ffn_up.bias", depth, Mh);
  m->wm_b_down = L.vec_stack("pred.blk.", "ffn_down.bias", depth, D);
  m->wm_norm_g = L.vec("pred.norm.weight", D);
  m->wm_norm_b = L.vec("pred.norm.bias", D);
  m->wm_b_p0 = L.vec("pred.proj.0.bias", Hq);
  m->wm_b_p2 = L.vec("pred.proj.2.bias", D);
  if (!L.dry && L.status == JEPA_B200_OK && wm_arena_maps(&a) != JEPA_B200_OK) L.status = JEPA_B200_ERR_CUDA;
}

extern "C" {

int jepa_b200_out_shape(const jepa_b200_model* m, int B, int pool, int64_t shape[3]) {
  if (!m || !shape || B < 1) return JEPA_B200_ERR_ARG;
  shape[0] = B;
  shape[1] = shape[2] = 0;
  switch (pool) {
    case JEPA_B200_POOL_NONE:
      shape[1] = m->N;
      shape[2] = m->cfg.dim;
      return 3;
    case JEPA_B200_POOL_MEAN:
      shape[1] = m->cfg.dim;
      return 2;
    case JEPA_B200_POOL_CLS:
      if (!m->cfg.has_cls) return JEPA_B200_ERR_ARG;
      shape[1] = m->cfg.dim;
      return 2;
    case JEPA_B200_POOL_ATTENTIVE:
      if (!m->has_head) return JEPA_B200_ERR_MISSING_TENSOR;
      shape[1] = m->cfg.n_classes;
      return 2;
    case JEPA_B200_POOL_LEWM:
      if (m->cfg.wm_depth < 1) return JEPA_B200_ERR_MISSING_TENSOR;
      shape[1] = m->cfg.dim;
      return 2;
    default:
      return JEPA_B200_ERR_ARG;
  }
}

int jepa_b200_encode(jepa_b200_model* m, const float* pixels, int B, int pool, float* out, size_t out_bytes,
                     void* stream) {
  int s = check_encode_args(m, pixels, B, pool, out, out_bytes);
  if (s) return s;
  DeviceGuard guard(m->device);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if ((s = ensure_workspace(m, B))) return s;
  m->have_timing = false;
  // The graph is captured when the same inputs come twice in a row (a call
  // with new buffers each time runs its kernels directly, capture-free), and
  // replayed while they stay the same; per-kernel events (profiling) need
  // the launches one by one.
  const EncodeKey key{pixels, out, B, pool, m->timeout_ns};
  const bool replay = m->use_graph && !m->prof && m->graph && key == m->g_key;
  const bool capture = m->use_graph && !m->prof && !replay && key == m->last_key;
  m->last_key = key;
  if (!replay && !capture) {
    m->launches = 0;
    if (cudaEventRecord(m->ev0, st) != cudaSuccess) return JEPA_B200_ERR_CUDA;
    if ((s = enqueue_forward(m, pixels, B, pool, out, st))) return s;
  } else {
    if (capture && (s = capture_forward(m, key))) return s;
    m->launches = m->g_launches;
    if (cudaEventRecord(m->ev0, st) != cudaSuccess) return JEPA_B200_ERR_CUDA;
    if (cudaGraphLaunch(m->graph, st) != cudaSuccess) return JEPA_B200_ERR_CUDA;
  }
  if (cudaEventRecord(m->ev1, st) != cudaSuccess) return JEPA_B200_ERR_CUDA;
  m->have_timing = true;
  return JEPA_B200_OK;
}

int jepa_b200_predict(jepa_b200_model* m, const float* tokens, int B, const int* ctx_idx, int n_ctx,
                      const int* tgt_idx, int n_tgt, float* out, size_t out_bytes, void* stream) {
  if (!m || !tokens || !ctx_idx || !tgt_idx || !out || B < 1 || n_ctx < 1 || n_tgt < 1) return JEPA_B200_ERR_ARG;
  if (m->cfg.pred_depth < 1) return JEPA_B200_ERR_ARG;
  if (n_ctx > m->N || n_tgt > m->N) return JEPA_B200_ERR_ARG;
  for (int i = 0; i < n_ctx; ++i)
    if (ctx_idx[i] < 0 || ctx_idx[i] >= m->N) return JEPA_B200_ERR_ARG;
  for (int i = 0; i < n_tgt; ++i)
    if (tgt_idx[i] < 0 || tgt_idx[i] >= m->N) return JEPA_B200_ERR_ARG;
  const long long rows = static_cast<long long>(B) * (n_ctx + n_tgt);
  if (rows * std::max(m->cfg.pred_mlp, 4096) >= (1ll << 31) ||
      static_cast<long long>(B) * m->N * m->cfg.dim >= (1ll << 31))
    return JEPA_B200_ERR_SHAPE;
  if (out_bytes < static_cast<size_t>(B) * n_tgt * m->cfg.dim * 4) return JEPA_B200_ERR_SHAPE;
  if ((reinterpret_cast<uintptr_t>(tokens) & 15) || (reinterpret_cast<uintptr_t>(out) & 15)) return JEPA_B200_ERR_ARG;
  DeviceGuard guard(m->device);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int L = n_ctx + n_tgt, Lpad = (L + 127) / 128 * 128;
  int s;
  if ((s = pred_workspace(m, static_cast<size_t>(rows), static_cast<size_t>(B) * n_ctx,
                          static_cast<size_t>(B) * n_tgt, static_cast<size_t>(B) * m->cfg.pred_heads * 64 * Lpad)))
    return s;
  // index lists, uploaded when they change (ctx at [0, N), tgt at [N, 2N))
  std::vector<int> h(static_cast<size_t>(2) * m->N, 0);
  std::copy(ctx_idx, ctx_idx + n_ctx, h.begin());
  std::copy(tgt_idx, tgt_idx + n_tgt, h.begin() + m->N);
  h.push_back(n_ctx);
  h.push_back(n_tgt);
  if (h != m->pidx_host) {
    if (cudaMemcpyAsync(m->pidx, h.data(), static_cast<size_t>(2) * m->N * sizeof(int), cudaMemcpyHostToDevice, st) !=
        cudaSuccess)
      return JEPA_B200_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return JEPA_B200_ERR_CUDA;  // h is a temporary
    m->pidx_host = h;
  }
  if (B != m->pops_B || n_ctx != m->pops_ctx || n_tgt != m->pops_tgt || tokens != m->pops_tokens ||
      out != m->pops_out) {
    m->pops_B = 0;
    if ((s = prepare_pred_ops(m, tokens, B, n_ctx, n_tgt, out))) return s;
    m->pops_B = B;
    m->pops_ctx = n_ctx;
    m->pops_tgt = n_tgt;
    m->pops_tokens = tokens;
    m->pops_out = out;
  }
  m->launches = 0;
  m->have_timing = false;
  if (cudaEventRecord(m->ev0, st) != cudaSuccess) return JEPA_B200_ERR_CUDA;
  if ((s = enqueue_predict(m, tokens, B, n_ctx, n_tgt, st))) return s;
  if (cudaEventRecord(m->ev1, st) != cudaSuccess) return JEPA_B200_ERR_CUDA;
  m->have_timing = true;
  return JEPA_B200_OK;
}

// One launch of the fused world-model kernel (steps 0: a predictor call).
static int wm_call(jepa_b200_model* m, const float* states, const float* actions, int C, int T0, int steps,
                   float* out, void* stream) {
  const jepa_b200_config& c = m->cfg;
  WmParams p{};
  p.D = c.dim;
  p.heads = c.wm_heads;
  p.mlp = c.wm_mlp;
  p.hq = c.wm_pred_hidden;
  p.A = c.wm_action_dim;
  p.window = c.wm_window;
  p.depth = c.wm_depth;
  p.T0 = T0;
  p.steps = steps;
  p.n_cand = C;
  p.n_act = steps > 0 ? T0 + steps - 1 : T0;
  p.eps = c.ln_eps;
  p.states = states;
  p.actions = actions;
  p.out = out;
  p.w_act0 = m->wm_w_act0;
  p.b_act0 = m->wm_b_act0;
  p.b_act2 = m->wm_b_act2;
  p.pos = m->wm_pos;
  p.b_ada = m->wm_b_ada;
  p.b_qkv = m->wm_b_qkv;
  p.b_out = m->wm_b_out;
  p.b_up = m->wm_b_up;
  p.b_down = m->wm_b_down;
  p.norm_g = m->wm_norm_g;
  p.norm_b = m->wm_norm_b;
  p.b_p0 = m->wm_b_p0;
  p.b_p2 = m->wm_b_p2;
  p.err = m->err;
  p.timeout_ns = m->timeout_ns;
  DeviceGuard guard(m->device);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  m->launches = 0;
  m->have_timing = false;
  if (cudaEventRecord(m->ev0, st) != cudaSuccess) return JEPA_B200_ERR_CUDA;
  int s = wm_launch(m->wm, p, st);
  if (s) return s;
  m->launches = 1;
  if (cudaEventRecord(m->ev1, st) != cudaSuccess) return JEPA_B200_ERR_CUDA;
  m->have_timing = true;
  return JEPA_B200_OK;
}

int jepa_b200_lewm_predict(jepa_b200_model* m, const float* states, const float* actions, int C, int T, float* out,
                           size_t out_bytes, void* stream) {
  if (!m || !states || !actions || !out || C < 1 || T < 1) return JEPA_B200_ERR_ARG;
  if (m->cfg.wm_depth < 1) return JEPA_B200_ERR_ARG;
  if (T > m->cfg.wm_window) return JEPA_B200_ERR_SHAPE;
  if (out_bytes < static_cast<size_t>(C) * T * m->cfg.dim * 4) return JEPA_B200_ERR_SHAPE;
  return wm_call(m, states, actions, C, T, 0, out, stream);
}

int jepa_b200_lewm_rollout(jepa_b200_model* m, const float* states, int T0, const float* actions, int C, int steps,
                           float* out, size_t out_bytes, void* stream) {
  if (!m || !states || !actions || !out || C < 1 || T0 < 1 || steps < 1) return JEPA_B200_ERR_ARG;
  if (m->cfg.wm_depth < 1) return JEPA_B200_ERR_ARG;
  if (out_bytes < static_cast<size_t>(C) * steps * m->cfg.dim * 4) return JEPA_B200_ERR_SHAPE;
  if (static_cast<long long>(C) * (T0 + steps) * m->cfg.dim >= (1ll << 40)) return JEPA_B200_ERR_SHAPE;
  return wm_call(m, states, actions, C, T0, steps, out, stream);
}

int jepa_b200_encode_host(jepa_b200_model* m, const float* pixels, int B, int pool, float* out, size_t out_bytes,
                          void* stream) {
  int s = check_encode_args(m, pixels, B, pool, out, out_bytes);
  if (s) return s;
  DeviceGuard guard(m->device);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const jepa_b200_config& c = m->cfg;
  const size_t pix_bytes = static_cast<size_t>(B) * c.frames * 3 * c.img_h * c.img_w * 4;
  const size_t res_bytes = out_elems(m, B, pool) * 4;
  if (pix_bytes > m->stage_pix_bytes) {
    cudaDeviceSynchronize();
    if (m->stage_pix) cudaFree(m->stage_pix);
    m->stage_pix = nullptr;
    m->stage_pix_bytes = 0;
    if (cudaMalloc(&m->stage_pix, pix_bytes) != cudaSuccess) return JEPA_B200_ERR_CUDA;
    m->stage_pix_bytes = pix_bytes;
  }
  if (res_bytes > m->stage_out_bytes) {
    cudaDeviceSynchronize();
    if (m->stage_out) cudaFree(m->stage_out);
    m->stage_out = nullptr;
    m->stage_out_bytes = 0;
    if (cudaMalloc(&m->stage_out, res_bytes) != cudaSuccess) return JEPA_B200_ERR_CUDA;
    m->stage_out_bytes = res_bytes;
  }
  if (cudaMemcpyAsync(m->stage_pix, pixels, pix_bytes, cudaMemcpyHostToDevice, st) != cudaSuccess)
    return JEPA_B200_ERR_CUDA;
  if ((s = jepa_b200_encode(m, m->stage_pix, B, pool, m->stage_out, res_bytes, stream))) return s;
  if (cudaMemcpyAsync(out, m->stage_out, res_bytes, cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return JEPA_B200_ERR_CUDA;
  return jepa_b200_sync_status(m, stream);
}

int jepa_b200_debug_stage(jepa_b200_model* m, const float* pixels, int B, int layer, int stage, float* out,
                          size_t out_bytes, void* stream) {
  if (!m || !pixels || !out || B < 1 || stage != 0) return JEPA_B200_ERR_ARG;
  if (layer < 0 || layer > m->cfg.depth) return JEPA_B200_ERR_ARG;
  const size_t need = static_cast<size_t>(B) * m->N * m->cfg.dim * 4;
  if (out_bytes < need) return JEPA_B200_ERR_SHAPE;
  DeviceGuard guard(m->device);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int s;
  if ((s = ensure_workspace(m, B))) return s;
  m->launches = 0;
  if ((s = run_embed_and_blocks(m, pixels, B, layer, st))) return s;
  if (cudaMemcpyAsync(out, m->X, need, cudaMemcpyDeviceToDevice, st) != cudaSuccess) return JEPA_B200_ERR_CUDA;
  return JEPA_B200_OK;
}

int jepa_b200_sync_status(jepa_b200_model* m, void* stream) {
  if (!m) return JEPA_B200_ERR_ARG;
  DeviceGuard guard(m->device);
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return JEPA_B200_ERR_CUDA;
  DevErr e{0, 0};
  if (cudaMemcpy(&e, m->err, sizeof(e), cudaMemcpyDeviceToHost) != cudaSuccess) return JEPA_B200_ERR_CUDA;
  if (e.code != DERR_NONE) {
    cudaMemset(m->err, 0, sizeof(DevErr));
    return e.code == DERR_TIMEOUT ? JEPA_B200_ERR_TIMEOUT : JEPA_B200_ERR_CUDA;
  }
  return JEPA_B200_OK;
}

double jepa_b200_last_ms(jepa_b200_model* m) {
  if (!m || !m->have_timing) return -1.0;
  DeviceGuard guard(m->device);
  if (cudaEventSynchronize(m->ev1) != cudaSuccess) return -1.0;
  float ms = 0.0f;
  if (cudaEventElapsedTime(&ms, m->ev0, m->ev1) != cudaSuccess) return -1.0;
  return ms;
}

size_t jepa_b200_model_n_bytes(const jepa_b200_model* m) { return m ? m->weight_bytes : 0; }

int jepa_b200_set_timeout_ns(jepa_b200_model* m, unsigned long long ns) {
  if (!m) return JEPA_B200_ERR_ARG;
  m->timeout_ns = ns;
  return JEPA_B200_OK;
}

int jepa_b200_set_graph(jepa_b200_model* m, int enable) {
  if (!m) return JEPA_B200_ERR_ARG;
  m->use_graph = enable != 0;
  return JEPA_B200_OK;
}

int jepa_b200_last_launch_count(const jepa_b200_model* m) { return m ? m->launches : -1; }

int jepa_b200_set_profiling(jepa_b200_model* m, int enable) {
  if (!m) return JEPA_B200_ERR_ARG;
  m->prof = enable != 0;
  return JEPA_B200_OK;
}

int jepa_b200_profile_read(jepa_b200_model* m, double* ms, int* launches, int n) {
  if (!m || !ms || !launches || n < JEPA_B200_KC_COUNT) return JEPA_B200_ERR_ARG;
  DeviceGuard guard(m->device);
  for (int i = 0; i < n; ++i) {
    ms[i] = 0.0;
    launches[i] = 0;
  }
  int s = JEPA_B200_OK;
  for (const auto& r : m->prof_recs) {
    float t = 0.0f;
    if (cudaEventSynchronize(m->prof_events[r.e1]) != cudaSuccess ||
        cudaEventElapsedTime(&t, m->prof_events[r.e0], m->prof_events[r.e1]) != cudaSuccess) {
      s = JEPA_B200_ERR_CUDA;
      continue;
    }
    ms[r.cls] += t;
    launches[r.cls] += 1;
  }
  m->prof_recs.clear();
  m->prof_used = 0;
  return s;
}

void jepa_b200_free(jepa_b200_model* m) {
  if (!m) return;
  DeviceGuard guard(m->device);
  cudaDeviceSynchronize();
  free_list(m->ws_allocs);
  free_list(m->pws_allocs);
  free_list(m->allocs);
  if (m->stage_pix) cudaFree(m->stage_pix);
  if (m->stage_out) cudaFree(m->stage_out);
  if (m->err) cudaFree(m->err);
  if (m->ev0) cudaEventDestroy(m->ev0);
  if (m->ev1) cudaEventDestroy(m->ev1);
  for (cudaEvent_t e : m->prof_events) cudaEventDestroy(e);
  if (m->graph) cudaGraphExecDestroy(m->graph);
  if (m->cap_stream) cudaStreamDestroy(m->cap_stream);
  delete m;
}

}  // extern "C"
