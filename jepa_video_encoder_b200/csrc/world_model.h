// Host-side declarations of the LeWM world model's fused kernel
// (world_model.cu), used by the loader and the entry points (model.cu).
#pragma once

#include "internal.h"

namespace jb {

// The LeWM world model's fused kernel (world_model.cu).  Weights in three
// 16-bit arenas by row length: D (action_embed.2, then per block adaLN [6D],
// attn_qkv [3D], attn_out [D], ffn_up [mlp]; then pred.proj.0 [hq]), mlp
// (ffn_down of every block) and hq (pred.proj.2).
struct WmArena {
  void* d = nullptr;
  void* m = nullptr;
  void* h = nullptr;
  int D = 0, mlp = 0, hq = 0, rows_d = 0, rows_m = 0, rows_h = 0, bf16 = 0;
  CUtensorMap tmD, tmM, tmH;
};
struct WmParams {
  int D, heads, mlp, hq, A, window, depth;
  int T0;      // observed frames per candidate
  int steps;   // 0: one predictor call over the T0 frames (every row out); else rollout steps
  int n_cand, cpc, n_act;
  float eps;
  const float* states;   // [n_cand, T0, D]
  const float* actions;  // [n_cand, n_act, A]
  float* out;            // [n_cand, T0, D] (steps 0) or [n_cand, steps, D]
  const float *w_act0, *b_act0, *b_act2, *pos;
  const float *b_ada, *b_qkv, *b_out, *b_up, *b_down;  // [depth, ...]
  const float *norm_g, *norm_b, *b_p0, *b_p2;
  DevErr* err;
  unsigned long long timeout_ns;
};
size_t wm_smem_bytes(int D, int mlp, int hq);
int wm_arena_maps(WmArena* a);
int wm_launch(const WmArena& a, const WmParams& p, cudaStream_t st);

}  // namespace jb
