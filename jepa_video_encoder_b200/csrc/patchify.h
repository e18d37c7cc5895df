// The patch-embed's input side (norm_pool.cu), used by the model and the
// single-kernel entry point.
#pragma once

#include "internal.h"

namespace jb {

// The unfolded patch matrix of a tubelet convolution, [B * n_patches, Kpad]
// in the 16-bit type (f16, or bf16): row = patch (clip, slot, patch row,
// patch column), column k = (c, dt, kh, kw) in the row-major order of a conv
// weight [D, 3, kt, p, p], columns past 3 kt p^2 zero.  It is the A operand
// of the patch-embed GEMM (EPI_PATCH).  a: device, 16-byte aligned.
int launch_patchify(const float* pixels, const PatchSrc& s, int B, int Kpad, void* a, cudaStream_t st, bool bf16);

}  // namespace jb
