// Internal interface of the tensor-core tier (nvfp4_gemv_tc.cu) for the C ABI in nvfp4_gemv.cu.
#ifndef NVFP4_TC_H
#define NVFP4_TC_H

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "nvfp4_prologue.h"

namespace nvfp4_tc {

using EncodeFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                              const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                              const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                              CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// K-splits of an N x K call (depends only on N, K and the SM count).
int choose_splits(int64_t n, int64_t k, int sms);
// Scratch bytes of a tier call of m rows (single or dual): fp32 partials (when K is split), an
// f16 copy of x, the rows' scales, and the dual's two fp32 results.
size_t scratch_bytes(int64_t n, int64_t k, int m, int sms);
// The tier's TMA scale boxes need K % 256 == 0 and 16-byte aligned scale codes.
bool usable(const void* s, int64_t k);
// Enqueue one call (arguments already checked as for nvfp4_gemv, 9 <= m <= 128), with x's
// prologue applied by the pass that makes its f16 copy.  The error word is the workspace's
// first int32; the scratch starts scratch_off bytes in.
int launch(EncodeFn encode, int sms, const uint8_t* w, const uint8_t* s, float g, const void* x,
           int64_t ldx, void* y, int64_t ldy, int m, int64_t n, int64_t k,
           const nvfp4_pro::Prologue& pro, void* ws, size_t ws_bytes, size_t scratch_off,
           cudaStream_t stream);
// The fused dual: o = bf16(silu(g_g W_gate x) * (g_u W_up x)), the two streams through the tier
// into fp32, then one combining pass.
int launch_dual(EncodeFn encode, int sms, const uint8_t* wg, const uint8_t* sg, float gg,
                const uint8_t* wu, const uint8_t* su, float gu, const void* x, int64_t ldx,
                void* y, int64_t ldy, int m, int64_t n, int64_t k, const nvfp4_pro::Prologue& pro,
                void* ws, size_t ws_bytes, size_t scratch_off, cudaStream_t stream);

// Several weights sharing x (nvfp4_gemv_multi): one x pass, then each weight through the tier
// as launch does it, so each output is bitwise that of its own launch.  The workspace must hold
// the largest scratch_bytes of the outputs.
int launch_multi(EncodeFn encode, int sms, const uint8_t* const* w, const uint8_t* const* s,
                 const float* g, void* const* y, const int64_t* ldy, const int64_t* n, int count,
                 const void* x, int64_t ldx, int m, int64_t k, const nvfp4_pro::Prologue& pro,
                 void* ws, size_t ws_bytes, size_t scratch_off, cudaStream_t stream);

}  // namespace nvfp4_tc

#endif
