// Weight-only NVFP4 GEMV / fused dual GEMV / multi-output GEMV for NVIDIA B200 (sm_100a), with
// its C ABI.
//
// The operation is the "w4a16_gemv" / "w4a16_gemv_dual" kernel family of a hybrid decoder's
// decode step ("Blueprint - circuit executor" page for qwen3.8-27b-nvfp4 on GB10, table
// "Kernels the plan launches"; weight format "nvfp4/g16", activations bf16, table "Weighted
// nodes"); the fused SiLU(gate)*up epilogue replaces that plan's separate "moe_silu_mul" launch
// (planner setting decode_split_silu).  The multi-output instance runs up to four weights that
// share x in one launch (that plan's two-output k/v and q+gate GEMVs).  Row counts 1..8 per pass
// (8-row speculative draft/verify round, kern-qwen38-sm103 model card, section "Run"); calls of
// up to 128 rows (the plan's multi_seq arms) run one pass per 8 rows.  Formats and the ABI are
// described in nvfp4.h.
//
// Design (B200-first):
//   * The path is HBM-bound: 0.5625 bytes per weight.  A persistent grid (one CTA per SM)
//     splits the work -- units of (RB output rows x 256 k) in row-group-major order -- into
//     equal contiguous ranges ("stream-K"), so every SM streams the same number of bytes.
//     Row groups cut by a range boundary are finished by the CTA holding their first unit
//     (the "owner", which reaches them last) after adding the other CTAs' fp32 partials in
//     CTA order; partials and flags live in a caller-provided workspace.  No data atomics:
//     the result is deterministic and the split depends only on (N, K, SM count), never on M.
//   * A producer warp streams each unit with TMA (cp.async.bulk.tensor, no multicast): one
//     RB-row x 128-byte box of packed weights per weight stream (128-byte swizzle) and, when
//     K % 256 == 0, one RB-row x 16-byte box of scale codes (otherwise the producer copies the
//     scale codes with cp.async).  Boxes past N or K are zero-filled.  Stages live in a ring of
//     shared memory guarded by mbarriers; the consumer warps decode and multiply.
//   * Decode in registers with the hardware conversions: cvt e2m1x2 -> f16x2 turns each byte
//     (two nibbles, k and k+1) into an f16 pair, cvt e4m3x2 -> f16x2 turns two scale codes into
//     f16, and one f16x2 multiply gives A = e2m1 * e4m3, exact in f16 (at most 6 significant
//     bits, magnitude in [2^-10, 2688] or zero).
//   * The dot products run on the tensor cores: mma.m16n8k16 (f16 in, fp32 accumulate) with
//     16 weight rows as A and x as B, padded to 8 columns (columns >= M are zero).  The same
//     instruction sequence serves every M, so row m of the output depends only on x row m:
//     bitwise row invariance across M = 1..8, and across 1..128 with the 8-row passes.  Within a
//     16-row tile the mma's row r is weight
//     row perm(r) (rows r and r+1 four apart), which makes the swizzled reads conflict-free.
//   * x is staged once per CTA in shared memory as f16 (cp.async, then converted in place,
//     each row by its own warps).  Each x row m is scaled by a power of two 2^e(m) chosen from
//     the row's largest magnitude in the CTA's k range (so it lands in [2^14, 2^15)); bf16
//     values convert exactly unless they are more than 2^31 times smaller than that maximum.
//     The partial sums are multiplied back by 2^-e(m) (exact) before they are combined.  The
//     producer issues at most kPrefetch units of weights before the consumers have requested
//     x: a longer queue of weight boxes ahead of those requests would delay them.
//   * Optional programmatic dependent launch: the weights stream in before the preceding
//     kernel on the stream has finished; x, y and the workspace are touched only after
//     griddepcontrol.wait.
//   * Epilogue in fp32: y = acc * g rounded to bf16; the dual computes
//     silu(g_g acc_g) * (g_u acc_u) with expf and rounds once.
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include "nvfp4.h"
#include "nvfp4_prologue.h"
#include "nvfp4_tc.h"

namespace {

// ------------------------------------------------------------------------------------------
// geometry

constexpr int kBlockK = 128;                 // k per mma block (4 lanes x 32) and per x slot
constexpr int kUnitK = 256;                  // k per unit (one stage)
constexpr int kWRowBytes = kUnitK / 2;       // 128 bytes of packed W per row and unit
constexpr int kSRowBytes = kUnitK / 16;      // 16 scale codes per row and unit
constexpr int kMaxRows = 256;                // tallest unit of any variant (TMA box limit)
constexpr int kSlotU4 = 16;                  // uint4 of x per 128-k block per row
constexpr int kRowPadU4 = 4;                 // 64-byte pad between x rows (bank offset)
constexpr int kSmemMax = 226 * 1024;
constexpr int kPartialFloats = kMaxRows * 8; // one stream's partial slot
constexpr int kSpinLimit = 1 << 24;          // bounded waits
constexpr int64_t kMaxK = int64_t(1) << 24;

// Launch geometry of each variant (build-time): consumer warps, 16-row tiles per warp, ring
// stages.  A unit is kRows = warps * tiles * 16 output rows by 256 k; a stage holds its W boxes
// (rows x 128 bytes per stream) followed by its scale boxes (rows x 16 bytes per stream).
#ifndef NVFP4_SINGLE_WARPS
#define NVFP4_SINGLE_WARPS 8
#define NVFP4_SINGLE_TILES 1
#endif
#ifndef NVFP4_DUAL_WARPS
#define NVFP4_DUAL_WARPS 8
#define NVFP4_DUAL_TILES 1
#endif
// The ring holds 4 to 8 stages: the row split of a launch is sized with the minimum, and a
// launch uses as many stages as its shared memory allows (the ring depth does not change
// the arithmetic).
constexpr int kMinStages = 4;
// Units of weights issued before the consumers have requested x (which may wait for the
// preceding kernel): a longer queue of weight boxes ahead of those requests delays them.
#ifndef NVFP4_PREFETCH_UNITS
#define NVFP4_PREFETCH_UNITS 2
#endif
constexpr int kPrefetch = NVFP4_PREFETCH_UNITS;
constexpr int kMaxStages = 8;
template <bool DUAL, int WARPS, int TILES>
struct Geo {
    static constexpr int kStreams = DUAL ? 2 : 1;
    static constexpr int kConsumerWarps = WARPS;
    static constexpr int kConsumers = WARPS * 32;
    static constexpr int kThreads = kConsumers + 32;           // + one producer warp
    static constexpr int kTiles = TILES;
    static constexpr int kRows = WARPS * TILES * 16;           // rows per unit
    static constexpr int kWBytes = kRows * kWRowBytes;         // W box per stream
    static constexpr int kSBytes = kRows * kSRowBytes;         // scale box per stream
    static constexpr int kStageBytes = kStreams * (kWBytes + kSBytes);
    static_assert(kRows <= kMaxRows, "unit taller than a TMA box / partial slot");
    static_assert(kStageBytes % 1024 == 0, "stages must keep 1024-byte alignment (swizzle)");
    static_assert(WARPS % 8 == 0, "x staging gives each of up to 8 x rows a whole warp");
};
template <bool DUAL> struct CfgSel;
template <> struct CfgSel<false> {
    using type = Geo<false, NVFP4_SINGLE_WARPS, NVFP4_SINGLE_TILES>;
};
template <> struct CfgSel<true> {
    using type = Geo<true, NVFP4_DUAL_WARPS, NVFP4_DUAL_TILES>;
};
template <bool DUAL> using Cfg = typename CfgSel<DUAL>::type;

enum ScaleMode { kScaleTma = 0, kScaleAsync8 = 1, kScaleScalar = 2 };

// Outputs of one launch of the single-stream kernel: several weight matrices with the same K
// share x, their row groups concatenated in output order (one output for nvfp4_gemv).  The dual
// kernel has one output fed by two weight streams (index = stream).
constexpr int kMaxOutputs = NVFP4_MAX_OUTPUTS;

struct Params {
    const uint8_t* s[kMaxOutputs];  // scale codes, per output (dual: per stream)
    float g[kMaxOutputs];           // global scales, per output (dual: per stream)
    uint16_t* y[kMaxOutputs];       // outputs (dual: y[0])
    int64_t ldy[kMaxOutputs];
    int64_t n[kMaxOutputs];         // rows of each output (dual: n[0])
    int64_t gend[kMaxOutputs];      // row groups of outputs 0..o together
    int outs;                       // outputs (1 for the dual)
    const uint16_t* x;
    int64_t ldx;
    int m;
    int64_t k;
    int ku;              // 256-k units along K (the last may be partial)
    int64_t units;       // row groups * ku
    int grid;
    int scale_mode;
    int stages;          // ring depth, kMinStages .. kMaxStages
    float* partial;      // [grid][2][kPartialFloats]
    uint32_t* flags;     // [grid]
    int32_t* error;
};

// Tensor maps of one launch: packed weights and scale codes per output (dual: per stream).
// A kernel instance carries only as many as it can use.
template <bool DUAL, bool MULTI>
struct Maps {
    static constexpr int kCount = DUAL ? 2 : (MULTI ? kMaxOutputs : 1);
    CUtensorMap w[kCount];
    CUtensorMap s[kCount];
};

// ------------------------------------------------------------------------------------------
// device helpers

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* b, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(b)), "r"(count));
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t* b, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(b)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* b) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(b)) : "memory");
}

// Bounded wait for the phase with the given parity to complete; false after the limit.
__device__ __forceinline__ bool mbar_wait(uint64_t* b, uint32_t parity) {
    const uint32_t a = smem_u32(b);
    for (int it = 0; it < kSpinLimit; ++it) {
        uint32_t done;
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(done)
            : "r"(a), "r"(parity)
            : "memory");
        if (done) return true;
    }
    return false;
}

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y,
                                            uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes "
        "[%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void named_barrier(int id, int count) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

__device__ __forceinline__ void cp_async16(void* dst, const void* src, bool valid) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src),
                 "r"(valid ? 16 : 0)
                 : "memory");
}

__device__ __forceinline__ void cp_async8(void* dst, const void* src, bool valid) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8, %2;" ::"r"(smem_u32(dst)), "l"(src),
                 "r"(valid ? 8 : 0)
                 : "memory");
}

// The mbarrier receives one arrival when all of this thread's earlier cp.async have landed.
__device__ __forceinline__ void cp_async_arrive(uint64_t* b) {
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(b))
                 : "memory");
}

__device__ __forceinline__ uint32_t hmul2(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// Two e4m3 scale codes (low byte = even group, high byte = odd group) -> f16x2, exact.
__device__ __forceinline__ uint32_t scale_pair(uint32_t codes) {
    uint32_t h;
    asm("{\n\t.reg .b16 t;\n\tcvt.u16.u32 t, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, t;\n\t}"
        : "=r"(h)
        : "r"(codes));
    return h;
}

__device__ __forceinline__ uint32_t bcast_lo(uint32_t v) { return __byte_perm(v, 0, 0x1010); }
__device__ __forceinline__ uint32_t bcast_hi(uint32_t v) { return __byte_perm(v, 0, 0x3232); }

// 8 e2m1 nibbles of a word (nibble i in bits 4i..4i+3, k order) -> 4 f16x2 words,
// p[i] = {lo: nibble 2i, hi: nibble 2i+1}, exact.
__device__ __forceinline__ void decode_word(uint32_t w, uint32_t (&p)[4]) {
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\tmov.b32 {b0, b1, b2, b3}, %4;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, b0;\n\tcvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %2, b2;\n\tcvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
        : "=r"(p[0]), "=r"(p[1]), "=r"(p[2]), "=r"(p[3])
        : "r"(w));
}

__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
        "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t ld_acquire(const uint32_t* p) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void st_release(uint32_t* p, uint32_t v) {
    asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ float4 ld_cg4(const float* p) {
    float4 r;
    asm volatile("ld.global.cg.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(r.x), "=f"(r.y), "=f"(r.z), "=f"(r.w)
                 : "l"(p));
    return r;
}

__device__ __forceinline__ uint16_t f2bf(float v) {
    uint32_t u;
    asm("{\n\t.reg .b16 h;\n\tcvt.rn.bf16.f32 h, %1;\n\tmov.b32 %0, {h, h};\n\t}"
        : "=r"(u)
        : "f"(v));
    return (uint16_t)u;
}

// A lane's decoded view of one stage for one stream: the multiply-ready k-step operands.
__device__ __forceinline__ void compute_tile(float (&acc)[2][4], uint4 wa, uint4 wb, uint32_t sca,
                                             uint32_t scb, const uint4 (&xv)[4]) {
    const uint32_t Sa = scale_pair(sca), Sb = scale_pair(scb);
    const uint32_t sa0 = bcast_lo(Sa), sa1 = bcast_hi(Sa);
    const uint32_t sb0 = bcast_lo(Sb), sb1 = bcast_hi(Sb);
    const uint32_t A[4] = {wa.x, wa.y, wa.z, wa.w};
    const uint32_t B[4] = {wb.x, wb.y, wb.z, wb.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        uint32_t pa[4], pb[4];
        decode_word(A[j], pa);
        decode_word(B[j], pb);
        const uint32_t sA = j < 2 ? sa0 : sa1, sB = j < 2 ? sb0 : sb1;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            pa[i] = hmul2(pa[i], sA);
            pb[i] = hmul2(pb[i], sB);
        }
        // k-step A: logical k {2q, 2q+1 | 2q+8, 2q+9} <- word k {0, 1 | 2, 3}
        mma16816(acc[0], pa[0], pb[0], pa[1], pb[1], xv[j].x, xv[j].y);
        // k-step B: word k {4, 5 | 6, 7}
        mma16816(acc[1], pa[2], pb[2], pa[3], pb[3], xv[j].z, xv[j].w);
    }
}


__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Row of the 16-row tile that the mma's row r (0..15) reads: rows r and r+1 of the fragment
// are four weight rows apart, so with the 128-byte swizzle the eight lanes of a quarter-warp
// touch eight distinct 16-byte bank groups.
__device__ __forceinline__ int perm_row(int r) { return (r & 8) | ((r >> 1) & 3) | ((r & 1) << 2); }

// Byte offset of 16-byte chunk c (0..7) of row r in a 128-byte-swizzled box of 128-byte rows.
__device__ __forceinline__ int swz(int r, int c) { return r * 128 + ((c ^ (r & 7)) << 4); }

// Write this lane's outputs of one tile of output o (rows ra, rb local to it): c0 (row ra,
// col 2q), c1 (ra, 2q+1), c2 (rb, 2q), c3 (rb, 2q+1).
__device__ __forceinline__ void store_tile(const Params& p, int o, int64_t ra, int64_t rb, int q,
                                           const float (&v)[4]) {
    const int c0 = 2 * q, c1 = 2 * q + 1;
    uint16_t* const y = p.y[o];
    const int64_t ldy = p.ldy[o], n = p.n[o];
    if (c0 < p.m) {
        if (ra < n) y[c0 * ldy + ra] = f2bf(v[0]);
        if (rb < n) y[c0 * ldy + rb] = f2bf(v[2]);
    }
    if (c1 < p.m) {
        if (ra < n) y[c1 * ldy + ra] = f2bf(v[1]);
        if (rb < n) y[c1 * ldy + rb] = f2bf(v[3]);
    }
}

// Output holding global row group rg (the groups of outputs 0..o end at p.gend[o]).
__device__ __forceinline__ int output_of(const Params& p, int64_t rg) {
    int o = 0;
    while (o + 1 < p.outs && rg >= p.gend[o]) ++o;
    return o;
}

// ------------------------------------------------------------------------------------------
// the kernel

// MULTI: the single-stream kernel over several outputs (nvfp4_gemv_multi); otherwise one output.
template <bool DUAL, bool MULTI>
__global__ void __launch_bounds__(Cfg<DUAL>::kThreads, 1)
    nvfp4_gemv_kernel(const Params p, const __grid_constant__ Maps<DUAL, MULTI> maps) {
    using C = Cfg<DUAL>;
    constexpr int NS = C::kStreams;
    const int S = p.stages;
    constexpr int kTiles = C::kTiles;
    constexpr int kRows = C::kRows;
    constexpr int kWBytes = C::kWBytes;
    constexpr int kSBytes = C::kSBytes;
    constexpr int kConsumerWarps = C::kConsumerWarps;
    constexpr int kConsumers = C::kConsumers;
    extern __shared__ __align__(16) uint8_t smem_raw[];
    // the ring starts on a 1024-byte boundary (the launch reserves the slack)
    uint8_t* const ring = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint4* const xsm = reinterpret_cast<uint4*>(ring + S * C::kStageBytes);
    __shared__ __align__(8) uint64_t full_bar[kMaxStages], empty_bar[kMaxStages], xreq_bar;
    __shared__ int s_amax[8];
    __shared__ float s_descale[8];

    pdl_launch_dependents();
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int cta = blockIdx.x;
    const int64_t U = p.units;
    const int64_t u_begin = U * cta / p.grid;
    const int64_t u_end = U * (cta + 1) / p.grid;
    if (u_begin >= u_end) return;
    const int ku = p.ku;
    const int64_t rg0 = u_begin / ku;
    const int b0 = (int)(u_begin - rg0 * ku);
    const int L = (int)(u_end - u_begin);
    const int uslots = L < ku ? L : ku;              // distinct 256-k units of the range
    const int xrow = 2 * uslots * kSlotU4 + kRowPadU4;  // uint4 per staged x row

    if (tid == 0) {
        // full: the expect_tx arrival, plus one per producer lane when the producer copies
        // the scale codes itself
        const uint32_t full_count = p.scale_mode == kScaleTma ? 1 : 1 + 32;
        for (int i = 0; i < kMaxStages; ++i) {
            mbar_init(&full_bar[i], full_count);
            mbar_init(&empty_bar[i], kConsumers);
        }
        mbar_init(&xreq_bar, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (tid < 8) s_amax[tid] = 0;
    __syncthreads();

    // ---- producer warp: stream the weight boxes and scale codes of every unit -------------
    // (weights and scales are not written by earlier work on the stream, so this may run
    // before griddepcontrol.wait)
    if (warp == kConsumerWarps) {
        const int mode = p.scale_mode;
        const uint32_t tx = NS * kWBytes + (mode == kScaleTma ? NS * kSBytes : 0);
        const int64_t srow = p.k >> 4;
        int64_t rg = rg0;
        int b = b0;
        // output of row group rg and its first row group (the single kernel's outputs follow
        // one another; the dual's two streams share one output)
        int o = MULTI ? output_of(p, rg0) : 0;
        int64_t gbase = o > 0 ? p.gend[o - 1] : 0;
        bool ok = true;
        int slot = 0;
        uint32_t phase = 0;  // parity of the ring pass in progress
        for (int i = 0; i < L; ++i) {
            if (i == kPrefetch) {
                // the rest of the ring queues behind the consumers' requests for x, which
                // would otherwise wait for every weight box issued before them
                if (lane == 0 && ok) ok = mbar_wait(&xreq_bar, 0);
                ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
                if (!ok) {
                    if (lane == 0) atomicExch(p.error, 2);
                    break;
                }
            }
            if (i >= S) {
                if (lane == 0 && ok) ok = mbar_wait(&empty_bar[slot], phase ^ 1u);
                ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
                if (!ok) {
                    if (lane == 0) atomicExch(p.error, 2);
                    break;
                }
            }
            uint8_t* dst = ring + slot * C::kStageBytes;
            uint8_t* sdst = dst + NS * kWBytes;
            const int y = (int)((rg - gbase) * kRows);  // first row of the unit in output o
            if (lane == 0) {
                mbar_expect_tx(&full_bar[slot], tx);
                tma_load_2d(dst, &maps.w[o], b * kWRowBytes, y, &full_bar[slot]);
                if constexpr (DUAL)
                    tma_load_2d(dst + kWBytes, &maps.w[1], b * kWRowBytes, y, &full_bar[slot]);
                if (mode == kScaleTma) {
                    tma_load_2d(sdst, &maps.s[o], b * kSRowBytes, y, &full_bar[slot]);
                    if constexpr (DUAL)
                        tma_load_2d(sdst + kSBytes, &maps.s[1], b * kSRowBytes, y, &full_bar[slot]);
                }
            }
            if (mode != kScaleTma) {
                // the 16 scale codes of each row for this unit (fewer in a ragged last unit)
#pragma unroll
                for (int s = 0; s < NS; ++s)
                    for (int r = lane; r < kRows; r += 32) {
                        const int64_t row = (int64_t)y + r;
                        const bool vrow = row < p.n[o];
                        const uint8_t* src = p.s[o + s] + (vrow ? row * srow : 0);
                        uint8_t* d = sdst + s * kSBytes + r * kSRowBytes;
                        const int64_t g0 = (int64_t)b * kSRowBytes;
                        if (mode == kScaleAsync8) {
                            cp_async8(d, src + (vrow ? g0 : 0), vrow && g0 < srow);
                            cp_async8(d + 8, src + (vrow && g0 + 8 < srow ? g0 + 8 : 0),
                                      vrow && g0 + 8 < srow);
                        } else {
                            for (int h = 0; h < 8; ++h) {
                                const bool v = vrow && g0 + 2 * h < srow;
                                *reinterpret_cast<uint16_t*>(d + 2 * h) =
                                    v ? *reinterpret_cast<const uint16_t*>(src + g0 + 2 * h)
                                      : (uint16_t)0;
                            }
                        }
                    }
                if (mode == kScaleAsync8) cp_async_arrive(&full_bar[slot]);
                else mbar_arrive(&full_bar[slot]);
            }
            if (++b == ku) {
                b = 0;
                ++rg;
                if (MULTI && o + 1 < p.outs && rg == p.gend[o]) gbase = p.gend[o++];
            }
            if (++slot == S) {
                slot = 0;
                phase ^= 1u;
            }
        }
        asm volatile("cp.async.wait_all;" ::: "memory");
        return;
    }

    // ---- consumers ------------------------------------------------------------------------
    const int g = lane >> 2, q = lane & 3;
    pdl_wait();  // x, y and the workspace may be produced / used by the preceding kernel

    // stage x (raw bf16) for the range's units (two 128-k blocks each, mod ku) with cp.async;
    // chunk (q, j) of a block-row holds k = blk*128 + 32q + 8j .. +8, stored at position
    // 4q + (j ^ q) so that the four lanes of a row read distinct banks
    const int kblocks = (int)((p.k + kBlockK - 1) / kBlockK);
    const int per_row = 2 * uslots * kSlotU4;
    for (int mm = 0; mm < p.m; ++mm)
        for (int c = tid; c < per_row; c += kConsumers) {
            const int xslot = c >> 4, qq = (c >> 2) & 3, jj = c & 3;
            int ub = b0 + (xslot >> 1);
            if (ub >= ku) ub -= ku;
            const int blk = 2 * ub + (xslot & 1);
            const int64_t kk = (int64_t)blk * kBlockK + 32 * qq + 8 * jj;
            const bool valid = blk < kblocks && kk < p.k;
            cp_async16(&xsm[mm * xrow + xslot * kSlotU4 + qq * 4 + (jj ^ qq)],
                       p.x + (valid ? mm * p.ldx + kk : 0), valid);
        }
    asm volatile("cp.async.commit_group;" ::: "memory");
    named_barrier(1, kConsumers);          // every consumer has issued its copies of x ...
    if (tid == 0) mbar_arrive(&xreq_bar);  // ... so the producer may queue the rest of the ring
    asm volatile("cp.async.wait_group 0;" ::: "memory");
    named_barrier(1, kConsumers);
    {
        // per-row largest magnitude, then conversion in place to f16 * 2^e(m): row r belongs
        // to the kConsumerWarps / mp warps w with w / (kConsumerWarps / mp) == r (mp = M
        // rounded up to a power of two), which share its amax through shared memory only
        // when there is more than one of them
        const int mp = p.m <= 1 ? 1 : (p.m <= 2 ? 2 : (p.m <= 4 ? 4 : 8));
        const int wpr = kConsumerWarps / mp;
        const int r = warp / wpr, part = warp - r * wpr;
        uint32_t a = 0;
        if (r < p.m)
            for (int c = part * 32 + lane; c < per_row; c += wpr * 32) {
                const uint4 v = xsm[r * xrow + c];
                // per-halfword maximum (two bf16 magnitudes per word), folded below
                a = __vmaxu2(a, __vmaxu2(__vmaxu2(v.x & 0x7FFF7FFFu, v.y & 0x7FFF7FFFu),
                                         __vmaxu2(v.z & 0x7FFF7FFFu, v.w & 0x7FFF7FFFu)));
            }
        a = max(a & 0xFFFFu, a >> 16);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) a = max(a, __shfl_xor_sync(0xFFFFFFFFu, a, o));
        if (wpr > 1) {
            if (lane == 0 && r < p.m) atomicMax(&s_amax[r], (int)a);
            named_barrier(1, kConsumers);
            a = r < p.m ? (uint32_t)s_amax[r] : 0u;
        }
        // a is the bf16 magnitude bit pattern of the row's largest |x| in the range; the scale
        // 2^e puts that maximum in [2^14, 2^15), inside f16's range
        int e = 0;
        if (a != 0u && a < 0x7F80u) e = 14 - ((int)(a >> 7) - 127);
        e = e > 126 ? 126 : (e < -126 ? -126 : e);
        const float sc = __uint_as_float((uint32_t)(e + 127) << 23);
        if (r < p.m) {
            if (part == 0 && lane == 0) s_descale[r] = __uint_as_float((uint32_t)(127 - e) << 23);
            for (int c = part * 32 + lane; c < per_row; c += wpr * 32) {
                const uint4 v = xsm[r * xrow + c];
                const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
                uint32_t h4[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const __half2 t = __floats2half2_rn(__uint_as_float(w4[i] << 16) * sc,
                                                        __uint_as_float(w4[i] & 0xFFFF0000u) * sc);
                    h4[i] = *reinterpret_cast<const uint32_t*>(&t);
                }
                xsm[r * xrow + c] = make_uint4(h4[0], h4[1], h4[2], h4[3]);
            }
        }
    }
    named_barrier(1, kConsumers);
    const float ds0 = 2 * q < p.m ? s_descale[2 * q] : 1.f;
    const float ds1 = 2 * q + 1 < p.m ? s_descale[2 * q + 1] : 1.f;

    // this lane's weight rows inside a tile (fragment rows g and g+8)
    const int pr_a = perm_row(g), pr_b = perm_row(g + 8);

    float acc[NS][kTiles][2][4];
#pragma unroll
    for (int s = 0; s < NS; ++s)
#pragma unroll
        for (int t = 0; t < kTiles; ++t)
#pragma unroll
            for (int h = 0; h < 2; ++h)
#pragma unroll
                for (int i = 0; i < 4; ++i) acc[s][t][h][i] = 0.f;

    float* const my_partial = p.partial + (int64_t)cta * 2 * kPartialFloats;
    int64_t cur_rg = rg0;
    int cur_b = b0, seg_b0 = b0;
    bool ok = true;
    int st = 0;
    uint32_t phase = 0;

#pragma unroll 1
    for (int i = 0; i < L; ++i) {
        int uslot = cur_b - b0;
        if (uslot < 0) uslot += ku;

        if (ok && !mbar_wait(&full_bar[st], phase)) {
            ok = false;
            atomicExch(p.error, 3);
        }
        const uint8_t* stage = ring + st * C::kStageBytes;
        const uint8_t* sstage = stage + NS * kWBytes;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            // the unit's two 128-k blocks: chunks 4h .. 4h+3 of each 128-byte row
            uint4 xv[4];
#pragma unroll
            for (int j = 0; j < 4; ++j)
                xv[j] = g < p.m ? xsm[g * xrow + (2 * uslot + h) * kSlotU4 + q * 4 + (j ^ q)]
                                : make_uint4(0, 0, 0, 0);
            uint4 wa[NS][kTiles], wb[NS][kTiles];
            uint32_t sa[NS][kTiles], sb[NS][kTiles];
#pragma unroll
            for (int s = 0; s < NS; ++s)
#pragma unroll
                for (int t = 0; t < kTiles; ++t) {
                    const int ra = (warp * kTiles + t) * 16 + pr_a;
                    const int rb = (warp * kTiles + t) * 16 + pr_b;
                    wa[s][t] = *reinterpret_cast<const uint4*>(stage + s * kWBytes + swz(ra, 4 * h + q));
                    wb[s][t] = *reinterpret_cast<const uint4*>(stage + s * kWBytes + swz(rb, 4 * h + q));
                    sa[s][t] = *reinterpret_cast<const uint16_t*>(sstage + s * kSBytes + ra * kSRowBytes + 8 * h + 2 * q);
                    sb[s][t] = *reinterpret_cast<const uint16_t*>(sstage + s * kSBytes + rb * kSRowBytes + 8 * h + 2 * q);
                }
            if (h == 1) mbar_arrive(&empty_bar[st]);
#pragma unroll
            for (int s = 0; s < NS; ++s)
#pragma unroll
                for (int t = 0; t < kTiles; ++t)
                    compute_tile(acc[s][t], wa[s][t], wb[s][t], sa[s][t], sb[s][t], xv);
        }

        if (cur_b + 1 == ku || i + 1 == L) {
            // ---- end of a row-group segment: units seg_b0 .. cur_b of row group cur_rg
            float tot[2][kTiles][4];
#pragma unroll
            for (int s = 0; s < NS; ++s)
#pragma unroll
                for (int t = 0; t < kTiles; ++t)
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        tot[s][t][e] = (acc[s][t][0][e] + acc[s][t][1][e]) * ((e & 1) ? ds1 : ds0);
                        acc[s][t][0][e] = 0.f;
                        acc[s][t][1][e] = 0.f;
                    }
            if (seg_b0 > 0) {
                // contributor: the row group started before this CTA's range
                if (2 * q < p.m) {
#pragma unroll
                    for (int s = 0; s < NS; ++s)
#pragma unroll
                        for (int t = 0; t < kTiles; ++t) {
                            float* dst = my_partial + s * kPartialFloats +
                                         ((warp * kTiles + t) * 32 + lane) * 4;
                            *reinterpret_cast<float4*>(dst) = make_float4(
                                tot[s][t][0], tot[s][t][1], tot[s][t][2], tot[s][t][3]);
                        }
                }
                named_barrier(1, kConsumers);
                // the release store orders every consumer's partial stores (ordered before it by
                // the barrier) ahead of the flag at GPU scope
                if (tid == 0) st_release(p.flags + cta, 1u);
            } else {
                if (cur_b + 1 != ku) {
                    // owner: the following CTAs hold the rest of this row group, each as the
                    // first segment of its range; wait for all of them at once, then add their
                    // partials in CTA order
                    int nc = 0;
                    while (cta + 1 + nc < p.grid &&
                           U * (cta + 1 + nc) / p.grid < (cur_rg + 1) * ku)
                        ++nc;
                    for (int c = tid; c < nc; c += kConsumers) {
                        const uint32_t* f = p.flags + cta + 1 + c;
                        int it = 0;
                        while (ld_acquire(f) == 0u && ++it < kSpinLimit) __nanosleep(20);
                        if (it >= kSpinLimit) atomicExch(p.error, 1);  // result invalid
                    }
                    named_barrier(1, kConsumers);
                    if (2 * q < p.m) {
                        for (int c = 0; c < nc; ++c) {
                            const float* src = p.partial + (int64_t)(cta + 1 + c) * 2 * kPartialFloats;
#pragma unroll
                            for (int s = 0; s < NS; ++s)
#pragma unroll
                                for (int t = 0; t < kTiles; ++t) {
                                    const float4 v = ld_cg4(src + s * kPartialFloats +
                                                            ((warp * kTiles + t) * 32 + lane) * 4);
                                    tot[s][t][0] += v.x;
                                    tot[s][t][1] += v.y;
                                    tot[s][t][2] += v.z;
                                    tot[s][t][3] += v.w;
                                }
                        }
                    }
                    named_barrier(1, kConsumers);
                    for (int c = tid; c < nc; c += kConsumers) p.flags[cta + 1 + c] = 0u;
                }
                const int o = MULTI ? output_of(p, cur_rg) : 0;
                const int64_t grow = (cur_rg - (o > 0 ? p.gend[o - 1] : 0)) * kRows;
#pragma unroll
                for (int t = 0; t < kTiles; ++t) {
                    const int64_t row0 = grow + (warp * kTiles + t) * 16;
                    float v[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        if (DUAL) {
                            const float a = tot[0][t][e] * p.g[0];
                            const float b = tot[1][t][e] * p.g[1];
                            v[e] = a / (1.0f + expf(-a)) * b;
                        } else {
                            v[e] = tot[0][t][e] * p.g[o];
                        }
                    }
                    store_tile(p, o, row0 + pr_a, row0 + pr_b, q, v);
                }
            }
            seg_b0 = 0;
        }
        if (++cur_b == ku) {
            cur_b = 0;
            ++cur_rg;
        }
        if (++st == S) {
            st = 0;
            phase ^= 1u;
        }
    }
}

// ------------------------------------------------------------------------------------------
// host side

struct DeviceInfo {
    int ok = -1;  // -1 unknown, 0 not a B200, 1 ok
    int sms = 0;
};
DeviceInfo g_dev[64];
// ------------------------------------------------------------------------------------------
// The input prologue as a pass of its own, ahead of the GEMV on the same stream: one CTA per row
// of x writes x' (and h).  A row-wide reduction (the RMS norm) cannot be split over the GEMV's
// CTAs without each of them reading the whole row (148 copies of it through L2 per launch) or a
// grid-wide barrier; one small grid chained by programmatic dependent launch costs less.  The
// arithmetic is that of nvfp4_prologue.h; thread t of a row takes 16-byte chunks t, t + 512, ...
// in order, then a fixed xor tree per warp and the warps in order.

constexpr int kProThreads = 512;
constexpr int kProKeep = 4;  // chunks a thread keeps in registers between the two passes

__global__ void __launch_bounds__(kProThreads)
    nvfp4_prologue_kernel(const nvfp4_pro::Prologue pro, const void* __restrict__ xv,
                          int64_t ldx, int64_t k, uint16_t* __restrict__ xo) {
    pdl_launch_dependents();
    pdl_wait();  // x and the prologue's arrays may come from the preceding kernel
    __shared__ float s_red[kProThreads / 32];
    __shared__ float s_inv;
    const int m = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (pro.kind == NVFP4_PROLOGUE_GATED_RMSNORM) {
        // x fp32: a warp per group of G channels (groups w, w + 16, ...); lane l holds elements
        // 4 (l + 32 i) .. +3 for i < G / 128, sums their squares in element order, then a fixed
        // xor tree over the warp
        const float* xr = static_cast<const float*>(xv) + m * ldx;
        const uint16_t* zr = pro.in + m * pro.ld_in;
        uint16_t* outr = xo + m * k;
        const int g = pro.group, q = g / 128;
        for (int64_t g0 = (int64_t)warp * g; g0 < k; g0 += (int64_t)(kProThreads / 32) * g) {
            float4 v[4];
            float ss = 0.f;
#pragma unroll
            for (int i = 0; i < 4; ++i)
                if (i < q) {
                    v[i] = *reinterpret_cast<const float4*>(xr + g0 + 4 * (lane + 32 * i));
                    ss = fmaf(v[i].x, v[i].x, ss);
                    ss = fmaf(v[i].y, v[i].y, ss);
                    ss = fmaf(v[i].z, v[i].z, ss);
                    ss = fmaf(v[i].w, v[i].w, ss);
                }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xFFFFFFFFu, ss, o);
            const float inv = nvfp4_pro::rms_inverse(ss, g, pro.eps);
#pragma unroll
            for (int i = 0; i < 4; ++i)
                if (i < q) {
                    const int e = 4 * (lane + 32 * i);
                    *reinterpret_cast<uint2*>(outr + g0 + e) = nvfp4_pro::gated_4(
                        v[i], *reinterpret_cast<const uint2*>(zr + g0 + e),
                        *reinterpret_cast<const uint2*>(pro.gamma + e), inv);
                }
        }
        return;
    }
    const uint16_t* const x = static_cast<const uint16_t*>(xv);
    const int64_t nch = k >> 3;
    const uint4* xr = reinterpret_cast<const uint4*>(x + m * ldx);
    const uint4* ar = reinterpret_cast<const uint4*>(pro.in + m * pro.ld_in);
    uint4* outr = reinterpret_cast<uint4*>(xo + m * k);
    constexpr int64_t kRound = (int64_t)kProKeep * kProThreads;
    if (pro.kind == NVFP4_PROLOGUE_SIGMOID_GATE) {
        for (int64_t base = 0; base < nch; base += kRound) {
            uint4 xv[kProKeep], tv[kProKeep];
#pragma unroll
            for (int u = 0; u < kProKeep; ++u) {
                const int64_t j = base + tid + u * kProThreads;
                if (j < nch) {
                    xv[u] = xr[j];
                    tv[u] = ar[j];
                }
            }
#pragma unroll
            for (int u = 0; u < kProKeep; ++u) {
                const int64_t j = base + tid + u * kProThreads;
                if (j < nch) outr[j] = nvfp4_pro::gate_8(xv[u], tv[u]);
            }
        }
        return;
    }
    const uint4* gr = reinterpret_cast<const uint4*>(pro.gamma);
    uint4* hr = pro.hout ? reinterpret_cast<uint4*>(pro.hout + m * pro.ldh) : nullptr;
    const bool keep = nch <= kRound;  // one round: h and gamma stay in registers
    uint4 hv[kProKeep], gv[kProKeep];
    float ss = 0.f;
    for (int64_t base = 0; base < nch; base += kRound) {
        uint4 xv[kProKeep], rv[kProKeep];
#pragma unroll
        for (int u = 0; u < kProKeep; ++u) {
            const int64_t j = base + tid + u * kProThreads;
            if (j < nch) {
                xv[u] = xr[j];
                rv[u] = ar[j];
                if (keep) gv[u] = gr[j];
            }
        }
#pragma unroll
        for (int u = 0; u < kProKeep; ++u) {
            const int64_t j = base + tid + u * kProThreads;
            if (j < nch) {
                hv[u] = nvfp4_pro::add_8(xv[u], rv[u]);
                ss = nvfp4_pro::sum_squares_8(hv[u], ss);
                if (hr) hr[j] = hv[u];
            }
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xFFFFFFFFu, ss, o);
    if (lane == 0) s_red[warp] = ss;
    __syncthreads();
    if (tid == 0) {
        float t = 0.f;
        for (int w = 0; w < kProThreads / 32; ++w) t += s_red[w];
        s_inv = nvfp4_pro::rms_inverse(t, k, pro.eps);
    }
    __syncthreads();
    const float inv = s_inv;
    if (keep) {
#pragma unroll
        for (int u = 0; u < kProKeep; ++u) {
            const int64_t j = tid + u * kProThreads;
            if (j < nch) outr[j] = nvfp4_pro::scale_8(hv[u], gv[u], inv);
        }
    } else {
        for (int64_t j = tid; j < nch; j += kProThreads)
            outr[j] = nvfp4_pro::norm_8(xr[j], ar[j], gr[j], inv);
    }
}

bool g_attr_set[3][64];  // single, dual, multi

using EncodeTiled = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                 const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                 const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                 CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiled g_encode = nullptr;

int device_info(int* dev_out, DeviceInfo** info) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
        cudaGetLastError();
        return NVFP4_ERR_ARCH;
    }
    DeviceInfo& di = g_dev[dev];
    if (di.ok < 0) {
        int major = 0, minor = 0, sms = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
            cudaGetLastError();
            return NVFP4_ERR_ARCH;
        }
        di.sms = sms;
        di.ok = (major == 10 && minor == 0) ? 1 : 0;
    }
    if (di.ok != 1) return NVFP4_ERR_ARCH;
    if (!g_encode) {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess || !fn) {
            cudaGetLastError();
            return NVFP4_ERR_ARCH;
        }
        g_encode = reinterpret_cast<EncodeTiled>(fn);
    }
    *dev_out = dev;
    *info = &di;
    return NVFP4_OK;
}

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// workspace: [error int32 | pad to 256][flags uint32[sms] | pad to 256][partials]
size_t workspace_layout(int sms, size_t* flags_off, size_t* partial_off) {
    *flags_off = 256;
    *partial_off = 256 + align_up((size_t)sms * 4, 256);
    return *partial_off + (size_t)sms * 2 * kPartialFloats * sizeof(float);
}

bool misaligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) != 0; }

int check_common(const void* x, int64_t ldx, const void* y, int64_t ldy, int m, int64_t n,
                 int64_t k, const void* ws, uint32_t flags, bool* noop) {
    *noop = false;
    if (flags & ~(uint32_t)(NVFP4_FLAG_PREFETCH_WEIGHTS | NVFP4_FLAG_WIDE_TENSOR))
        return NVFP4_ERR_SHAPE;
    if (m < 0 || m > NVFP4_MAX_ROWS) return NVFP4_ERR_ROWS;
    if (n < 0 || k < 0 || (k % 32) != 0 || k > kMaxK) return NVFP4_ERR_SHAPE;
    if (m == 0 || n == 0) {
        *noop = true;
        return NVFP4_OK;
    }
    if (n > (int64_t(1) << 31) - kMaxRows) return NVFP4_ERR_SHAPE;
    if (ldy < n) return NVFP4_ERR_SHAPE;
    if (k > 0 && ldx < k) return NVFP4_ERR_SHAPE;
    if (!y || (k > 0 && !x)) return NVFP4_ERR_NULL;
    if (k > 0 && ((ldx % 8) != 0 || misaligned(x, 16))) return NVFP4_ERR_ALIGN;
    if (misaligned(y, 2)) return NVFP4_ERR_ALIGN;
    if (!ws || misaligned(ws, 16)) return NVFP4_ERR_WORKSPACE;
    return NVFP4_OK;
}

int check_weight(const uint8_t* w, const uint8_t* s) {
    if (!w || !s) return NVFP4_ERR_NULL;
    if (misaligned(w, 16) || misaligned(s, 2)) return NVFP4_ERR_ALIGN;
    return NVFP4_OK;
}

// Bytes [lo, hi) spanned by m rows of `cols` bf16 values at row stride ld (m, cols > 0).
struct Range {
    uintptr_t lo, hi;
};

Range rows_range(const void* p, int m, int64_t ld, int64_t cols) {
    const uintptr_t lo = reinterpret_cast<uintptr_t>(p);
    return {lo, lo + (uintptr_t)(((int64_t)(m - 1) * ld + cols) * 2)};
}

bool overlap(Range a, Range b) { return a.lo < b.hi && b.lo < a.hi; }

// A caller's prologue checked against the call's x (M x K) and its outputs `ys`, turned into
// the kernels' form (kind NONE for NULL).
int check_pro(const nvfp4_prologue_t* pp, const void* x, int64_t ldx, int m, int64_t k,
              const Range* ys, int ny, nvfp4_pro::Prologue* out) {
    memset(out, 0, sizeof(*out));
    if (!pp || pp->kind == NVFP4_PROLOGUE_NONE) return NVFP4_OK;
    if (pp->kind == NVFP4_PROLOGUE_GATED_RMSNORM) {
        // x is fp32 here: check_common's 16-byte rows and ldx % 8 hold for it too
        const int g = pp->group;
        if (!(pp->eps >= 0.0f && pp->eps <= 3.402823466e38f)) return NVFP4_ERR_SHAPE;
        if (g < 128 || g > 512 || (g % 128) != 0) return NVFP4_ERR_SHAPE;
        out->kind = pp->kind;
        out->eps = pp->eps;
        out->group = g;
        if (m <= 0 || k <= 0) return NVFP4_OK;
        if ((k % g) != 0 || pp->ld_gate < k) return NVFP4_ERR_SHAPE;
        if (!pp->gate || !pp->gamma) return NVFP4_ERR_NULL;
        if ((pp->ld_gate % 8) != 0 || misaligned(pp->gate, 16) || misaligned(pp->gamma, 16))
            return NVFP4_ERR_ALIGN;
        out->in = static_cast<const uint16_t*>(pp->gate);
        out->ld_in = pp->ld_gate;
        out->gamma = static_cast<const uint16_t*>(pp->gamma);
        return NVFP4_OK;
    }
    const bool norm = pp->kind == NVFP4_PROLOGUE_ADD_RMSNORM;
    if (!norm && pp->kind != NVFP4_PROLOGUE_SIGMOID_GATE) return NVFP4_ERR_SHAPE;
    if (norm && !(pp->eps >= 0.0f && pp->eps <= 3.402823466e38f)) return NVFP4_ERR_SHAPE;
    out->kind = pp->kind;
    out->eps = norm ? pp->eps : 0.0f;
    if (m <= 0 || k <= 0) return NVFP4_OK;  // nothing to read or write
    const void* in = norm ? pp->residual : pp->gate;
    const int64_t ld_in = norm ? pp->ld_residual : pp->ld_gate;
    void* hout = norm ? pp->residual_out : nullptr;
    if (!in || (norm && !pp->gamma)) return NVFP4_ERR_NULL;
    if (ld_in < k || (hout && pp->ld_residual_out < k)) return NVFP4_ERR_SHAPE;
    if ((ld_in % 8) != 0 || misaligned(in, 16) || (norm && misaligned(pp->gamma, 16)))
        return NVFP4_ERR_ALIGN;
    if (hout && ((pp->ld_residual_out % 8) != 0 || misaligned(hout, 16))) return NVFP4_ERR_ALIGN;
    // residual_out is written while other CTAs read x, residual and gamma; y is written while
    // they read the residual or the gate
    const Range rin = rows_range(in, m, ld_in, k);
    for (int i = 0; i < ny; ++i)
        if (overlap(rin, ys[i])) return NVFP4_ERR_ALIAS;
    if (hout) {
        const Range ro = rows_range(hout, m, pp->ld_residual_out, k);
        if (overlap(ro, rows_range(x, m, ldx, k)) || overlap(ro, rin) ||
            overlap(ro, rows_range(pp->gamma, 1, k, k)))
            return NVFP4_ERR_ALIAS;
        for (int i = 0; i < ny; ++i)
            if (overlap(ro, ys[i])) return NVFP4_ERR_ALIAS;
    }
    out->in = static_cast<const uint16_t*>(in);
    out->ld_in = ld_in;
    out->gamma = norm ? static_cast<const uint16_t*>(pp->gamma) : nullptr;
    out->hout = static_cast<uint16_t*>(hout);
    out->ldh = hout ? pp->ld_residual_out : 0;
    return NVFP4_OK;
}


// 2-D map over a [rows][cols] byte matrix with row stride = cols: box = box_cols bytes x
// box_rows rows, zero fill outside.
bool encode_map(CUtensorMap* map, const uint8_t* base, int64_t rows, int64_t cols, int box_cols,
                int box_rows, CUtensorMapSwizzle swizzle) {
    const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)cols};
    const cuuint32_t box[2] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return g_encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(base), dims,
                    strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// One output of a launch: its weight streams (two for the dual, gate then up), their global
// scales, and its rows.
struct Span {
    const uint8_t* w[2];
    const uint8_t* s[2];
    float g[2];
    void* y;
    int64_t ldy;
    int64_t n;
};

constexpr size_t kXSlotBytes = (size_t)2 * kSlotU4 * 16;  // staged x per unit per row: 512 B

// Row groups one launch may hold for this K, or -1 for no limit: the staged x of a CTA's range
// (M rows x the range's 256-k units, sized for M = 8 so that the split never depends on M) must
// fit shared memory beside the smallest ring.
template <bool DUAL>
int64_t max_groups_per_launch(int64_t k, int sms) {
    using C = Cfg<DUAL>;
    const int ku = (int)((k + kUnitK - 1) / kUnitK);
    const size_t mx = NVFP4_PASS_ROWS;
    const int64_t max_slots = (int64_t)((kSmemMax - 1024 - kMinStages * C::kStageBytes -
                                         mx * kRowPadU4 * 16) /
                                        (mx * kXSlotBytes));
    if (max_slots >= ku) return -1;
    const int64_t groups = (int64_t)sms * max_slots / ku;
    return groups > 0 ? groups : 1;
}

// One launch over the spans' row groups, concatenated in order (the dual takes one span; more
// than one span needs MULTI).
template <bool DUAL, bool MULTI>
int launch_spans(const Span* sp, int count, const void* x, int64_t ldx, int m, int64_t k,
                 void* ws, size_t ws_bytes, uint32_t flags, cudaStream_t stream) {
    using C = Cfg<DUAL>;
    static_assert(!(DUAL && MULTI), "the dual kernel has one output");
    if (count > Maps<DUAL, MULTI>::kCount / (DUAL ? 2 : 1)) return NVFP4_ERR_SHAPE;
    if (m > NVFP4_PASS_ROWS) {
        // more rows than one pass: consecutive blocks of NVFP4_PASS_ROWS rows of x and y, one
        // launch each, in stream order on the same workspace; every row is computed exactly
        // as in a call of its own block, so rows stay bitwise invariant over M
        for (int r0 = 0; r0 < m; r0 += NVFP4_PASS_ROWS) {
            Span part[kMaxOutputs];
            for (int o = 0; o < count; ++o) {
                part[o] = sp[o];
                part[o].y = static_cast<uint16_t*>(sp[o].y) + (int64_t)r0 * sp[o].ldy;
            }
            const int rows = m - r0 < NVFP4_PASS_ROWS ? m - r0 : NVFP4_PASS_ROWS;
            const int st = launch_spans<DUAL, MULTI>(
                part, count, static_cast<const uint16_t*>(x) + (int64_t)r0 * ldx, ldx, rows, k,
                ws, ws_bytes, flags, stream);
            if (st != NVFP4_OK) return st;
        }
        return NVFP4_OK;
    }
    constexpr int NS = C::kStreams;
    int dev = 0;
    DeviceInfo* di = nullptr;
    int st = device_info(&dev, &di);
    if (st != NVFP4_OK) return st;
    size_t flags_off, partial_off;
    const size_t need = workspace_layout(di->sms, &flags_off, &partial_off);
    if (ws_bytes < need) return NVFP4_ERR_WORKSPACE;

    if (k == 0) {  // empty sum: y = 0 (silu(0) * 0 = 0 for the dual)
        for (int o = 0; o < count; ++o)
            if (cudaMemset2DAsync(sp[o].y, (size_t)sp[o].ldy * 2, 0, (size_t)sp[o].n * 2,
                                  (size_t)m, stream) != cudaSuccess) {
                cudaGetLastError();
                return NVFP4_ERR_LAUNCH;
            }
        return NVFP4_OK;
    }

    const int variant = DUAL ? 1 : (MULTI ? 2 : 0);
    if (!g_attr_set[variant][dev]) {
        if (cudaFuncSetAttribute(nvfp4_gemv_kernel<DUAL, MULTI>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemMax) !=
            cudaSuccess) {
            cudaGetLastError();
            return NVFP4_ERR_LAUNCH;
        }
        g_attr_set[variant][dev] = true;
    }

    // how the producer moves the scale codes: TMA needs 16-byte aligned scale rows
    int scale_mode = kScaleTma;
    for (int o = 0; o < count; ++o)
        for (int i = 0; i < NS; ++i)
            if ((k % kUnitK) != 0 || misaligned(sp[o].s[i], 16)) scale_mode = kScaleAsync8;
    if (scale_mode == kScaleAsync8) {
        for (int o = 0; o < count; ++o)
            for (int i = 0; i < NS; ++i)
                if ((k % kBlockK) != 0 || misaligned(sp[o].s[i], 8)) scale_mode = kScaleScalar;
    }

    const int ku = (int)((k + kUnitK - 1) / kUnitK);
    Params p;
    memset(&p, 0, sizeof(p));
    Maps<DUAL, MULTI> maps;
    memset(&maps, 0, sizeof(maps));
    int64_t groups = 0;
    for (int o = 0; o < count; ++o) {
        const Span& a = sp[o];
        // map / pointer slot of output o (single) or of stream i (dual)
        for (int i = 0; i < NS; ++i) {
            const int slot = DUAL ? i : o;
            p.s[slot] = a.s[i];
            p.g[slot] = a.g[i];
            if (!encode_map(&maps.w[slot], a.w[i], a.n, k / 2, kWRowBytes, C::kRows,
                            CU_TENSOR_MAP_SWIZZLE_128B))
                return NVFP4_ERR_LAUNCH;
            if (scale_mode == kScaleTma &&
                !encode_map(&maps.s[slot], a.s[i], a.n, k / 16, kSRowBytes, C::kRows,
                            CU_TENSOR_MAP_SWIZZLE_NONE))
                return NVFP4_ERR_LAUNCH;
        }
        p.y[o] = static_cast<uint16_t*>(a.y);
        p.ldy[o] = a.ldy;
        p.n[o] = a.n;
        groups += (a.n + C::kRows - 1) / C::kRows;
        p.gend[o] = groups;
    }
    p.outs = count;
    p.x = static_cast<const uint16_t*>(x);
    p.ldx = ldx;
    p.m = m;
    p.k = k;
    p.ku = ku;
    p.units = groups * ku;
    const int max_grid = di->sms;
    p.grid = (int)(p.units < max_grid ? p.units : max_grid);
    p.scale_mode = scale_mode;
    char* wsb = static_cast<char*>(ws);
    p.partial = reinterpret_cast<float*>(wsb + partial_off);
    p.flags = reinterpret_cast<uint32_t*>(wsb + flags_off);
    p.error = reinterpret_cast<int32_t*>(wsb);
    const int64_t max_range = (p.units + p.grid - 1) / p.grid;
    const int slots = (int)(max_range < ku ? max_range : ku);
    const size_t xbytes = (size_t)m * ((size_t)slots * kXSlotBytes + kRowPadU4 * 16);
    int stages = (int)((kSmemMax - 1024 - xbytes) / C::kStageBytes);
    stages = stages > kMaxStages ? kMaxStages : stages;
    if (stages < kMinStages) return NVFP4_ERR_LAUNCH;  // cannot happen: the split bounds x
    p.stages = stages;
    const size_t smem = 1024 + (size_t)stages * C::kStageBytes + xbytes;

    cudaLaunchConfig_t cfg;
    memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = dim3(p.grid);
    cfg.blockDim = dim3(C::kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    if (flags & NVFP4_FLAG_PREFETCH_WEIGHTS) {
        cfg.attrs = attr;
        cfg.numAttrs = 1;
    }
    if (cudaLaunchKernelEx(&cfg, nvfp4_gemv_kernel<DUAL, MULTI>, p, maps) != cudaSuccess) {
        cudaGetLastError();
        return NVFP4_ERR_LAUNCH;
    }
    return NVFP4_OK;
}

// One output (one or two weight streams), split into launches of at most
// max_groups_per_launch row groups.
template <bool DUAL>
int launch(const uint8_t* const* w, const uint8_t* const* s, const float* gs, const void* x,
           int64_t ldx, void* y, int64_t ldy, int m, int64_t n, int64_t k, void* ws,
           size_t ws_bytes, uint32_t flags, cudaStream_t stream) {
    using C = Cfg<DUAL>;
    constexpr int NS = C::kStreams;
    int dev = 0;
    DeviceInfo* di = nullptr;
    int st = device_info(&dev, &di);
    if (st != NVFP4_OK) return st;
    const int64_t cap = max_groups_per_launch<DUAL>(k, di->sms);
    const int64_t rows_per_launch = cap < 0 ? n : cap * C::kRows;
    for (int64_t r0 = 0; r0 < n; r0 += rows_per_launch) {
        Span a;
        memset(&a, 0, sizeof(a));
        for (int i = 0; i < NS; ++i) {
            a.w[i] = w[i] + r0 * (k / 2);
            a.s[i] = s[i] + r0 * (k / 16);
            a.g[i] = gs[i];
        }
        a.y = static_cast<uint16_t*>(y) + r0;
        a.ldy = ldy;
        a.n = (n - r0) < rows_per_launch ? (n - r0) : rows_per_launch;
        if ((st = launch_spans<DUAL, false>(&a, 1, x, ldx, m, k, ws, ws_bytes, flags, stream)) !=
            NVFP4_OK)
            return st;
    }
    return NVFP4_OK;
}

// Bytes the prologue pass adds after the workspace layout: x' of m rows, row stride k.
size_t prologue_scratch_bytes(int m, int64_t k) {
    return ((size_t)m * (size_t)k * 2 + 255) / 256 * 256;
}

// Enqueues the prologue pass of a call, when it has one, and points x / ldx at its output
// (x' in the workspace after its layout).  Nothing is enqueued when the workspace is short.
int prologue_pass(const nvfp4_pro::Prologue& pro, const void** x, int64_t* ldx, int m, int64_t k,
                  void* ws, size_t ws_bytes, uint32_t flags, cudaStream_t stream) {
    if (pro.kind == NVFP4_PROLOGUE_NONE || m == 0 || k == 0) return NVFP4_OK;
    int dev = 0;
    DeviceInfo* di = nullptr;
    int st = device_info(&dev, &di);
    if (st != NVFP4_OK) return st;
    size_t flags_off, partial_off;
    const size_t base = workspace_layout(di->sms, &flags_off, &partial_off);
    if (ws_bytes < base + prologue_scratch_bytes(m, k)) return NVFP4_ERR_WORKSPACE;
    uint16_t* xo = reinterpret_cast<uint16_t*>(static_cast<char*>(ws) + base);
    cudaLaunchConfig_t cfg;
    memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = dim3((unsigned)m);
    cfg.blockDim = dim3(kProThreads);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    if (flags & NVFP4_FLAG_PREFETCH_WEIGHTS) {
        cfg.attrs = attr;
        cfg.numAttrs = 1;
    }
    if (cudaLaunchKernelEx(&cfg, nvfp4_prologue_kernel, pro, *x, *ldx, k, xo) != cudaSuccess) {
        cudaGetLastError();
        return NVFP4_ERR_LAUNCH;
    }
    *x = xo;
    *ldx = k;
    return NVFP4_OK;
}

}  // namespace

// ------------------------------------------------------------------------------------------
// Scratch of nvfp4_gemv_noalloc: the workspace of nvfp4_gemv (error word, one flag per CTA,
// one pair of partial tiles per CTA, in workspace_layout's order) compiled into the library
// for grids of up to kNoAllocSms CTAs, so that the call needs no buffer from its caller.

constexpr int kNoAllocSms = 160;
constexpr size_t kNoAllocFlagsBytes = ((size_t)kNoAllocSms * 4 + 255) / 256 * 256;
constexpr size_t kNoAllocBytes =
    256 + kNoAllocFlagsBytes + (size_t)kNoAllocSms * 2 * kPartialFloats * sizeof(float);
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocBytes];

namespace {
void* g_noalloc_ptr[64];  // the array's device address, per device, found at the first call
}  // namespace

// ------------------------------------------------------------------------------------------
// C ABI

extern "C" {

int nvfp4_pack_info(int64_t n, int64_t k, nvfp4_pack_info_t* out) {
    if (!out) return NVFP4_ERR_NULL;
    if (n < 0 || k < 0 || (k % 32) != 0) return NVFP4_ERR_SHAPE;
    memset(out, 0, sizeof(*out));
    out->n = n;
    out->k = k;
    out->weight_bytes = n * (k / 2);
    out->scale_bytes = n * (k / 16);
    out->weight_row_bytes = k / 2;
    out->scale_row_bytes = k / 16;
    out->group = NVFP4_GROUP;
    out->max_rows = NVFP4_MAX_ROWS;
    out->align_bytes = 16;
    out->layout_version = NVFP4_LAYOUT_VERSION;
    return NVFP4_OK;
}

int nvfp4_workspace_bytes(size_t* bytes) {
    if (!bytes) return NVFP4_ERR_NULL;
    int dev = 0;
    DeviceInfo* di = nullptr;
    int st = device_info(&dev, &di);
    if (st != NVFP4_OK) return st;
    size_t a, b;
    *bytes = workspace_layout(di->sms, &a, &b);
    return NVFP4_OK;
}

int nvfp4_gemv_pro(const nvfp4_prologue_t* prologue, const uint8_t* w, const uint8_t* s,
                   float global_scale, const void* x, int64_t ldx, void* y, int64_t ldy, int m,
                   int64_t n, int64_t k, void* workspace, size_t workspace_bytes, uint32_t flags,
                   cudaStream_t stream) {
    bool noop = false;
    int st = check_common(x, ldx, y, ldy, m, n, k, workspace, flags, &noop);
    if (st != NVFP4_OK) return st;
    nvfp4_pro::Prologue pro;
    const Range yr = noop ? Range{0, 0} : rows_range(y, m, ldy, n);
    if ((st = check_pro(prologue, x, ldx, m, k, &yr, noop ? 0 : 1, &pro)) != NVFP4_OK) return st;
    if (noop) return NVFP4_OK;
    if (k > 0 && (st = check_weight(w, s)) != NVFP4_OK) return st;
    if ((flags & NVFP4_FLAG_WIDE_TENSOR) && m > NVFP4_PASS_ROWS && k > 0 &&
        pro.kind != NVFP4_PROLOGUE_GATED_RMSNORM && nvfp4_tc::usable(s, k)) {
        int dev = 0;
        DeviceInfo* di = nullptr;
        if ((st = device_info(&dev, &di)) != NVFP4_OK) return st;
        size_t flags_off, partial_off;
        const size_t base = workspace_layout(di->sms, &flags_off, &partial_off);
        return nvfp4_tc::launch(g_encode, di->sms, w, s, global_scale, x, ldx, y, ldy, m, n, k,
                                pro, workspace, workspace_bytes, base, stream);
    }
    if ((st = prologue_pass(pro, &x, &ldx, m, k, workspace, workspace_bytes, flags, stream)) !=
        NVFP4_OK)
        return st;
    const uint8_t* ws_[1] = {w};
    const uint8_t* ss_[1] = {s};
    const float gs[1] = {global_scale};
    return launch<false>(ws_, ss_, gs, x, ldx, y, ldy, m, n, k, workspace, workspace_bytes,
                         flags, stream);
}

int nvfp4_gemv_ex(const uint8_t* w, const uint8_t* s, float global_scale, const void* x,
                  int64_t ldx, void* y, int64_t ldy, int m, int64_t n, int64_t k,
                  void* workspace, size_t workspace_bytes, uint32_t flags, cudaStream_t stream) {
    return nvfp4_gemv_pro(nullptr, w, s, global_scale, x, ldx, y, ldy, m, n, k, workspace,
                          workspace_bytes, flags, stream);
}

int nvfp4_gemv(const uint8_t* w, const uint8_t* s, float global_scale, const void* x,
               int64_t ldx, void* y, int64_t ldy, int m, int64_t n, int64_t k, void* workspace,
               size_t workspace_bytes, cudaStream_t stream) {
    return nvfp4_gemv_pro(nullptr, w, s, global_scale, x, ldx, y, ldy, m, n, k, workspace,
                          workspace_bytes, 0u, stream);
}

int nvfp4_gemv_noalloc(const uint8_t* w, const uint8_t* s, float global_scale, const void* x,
                       int64_t ldx, void* y, int64_t ldy, int m, int64_t n, int64_t k,
                       cudaStream_t stream) {
    bool noop = false;
    // check_common also vets a caller's workspace pointer; hand it a stand-in, the scratch's
    // size is checked against the device below.
    alignas(16) static const unsigned char stand_in[16] = {0};
    int st = check_common(x, ldx, y, ldy, m, n, k, stand_in, 0u, &noop);
    if (st != NVFP4_OK || noop) return st;
    if (k > 0 && (st = check_weight(w, s)) != NVFP4_OK) return st;
    int dev = 0;
    DeviceInfo* di = nullptr;
    if ((st = device_info(&dev, &di)) != NVFP4_OK) return st;
    size_t flags_off, partial_off;
    if (workspace_layout(di->sms, &flags_off, &partial_off) > kNoAllocBytes)
        return NVFP4_ERR_WORKSPACE;  // more SMs than the compiled-in scratch covers
    if (!g_noalloc_ptr[dev]) {
        void* ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || !ptr) {
            cudaGetLastError();
            return NVFP4_ERR_LAUNCH;
        }
        g_noalloc_ptr[dev] = ptr;
    }
    void* scratch = g_noalloc_ptr[dev];
    // The previous call left its error word and flags behind; start this one from zero.
    if (cudaMemsetAsync(scratch, 0, partial_off, stream) != cudaSuccess) {
        cudaGetLastError();
        return NVFP4_ERR_LAUNCH;
    }
    const uint8_t* ws_[1] = {w};
    const uint8_t* ss_[1] = {s};
    const float gs[1] = {global_scale};
    return launch<false>(ws_, ss_, gs, x, ldx, y, ldy, m, n, k, scratch, kNoAllocBytes, 0u,
                         stream);
}

int nvfp4_gemv_dual_pro(const nvfp4_prologue_t* prologue, const uint8_t* w_gate,
                        const uint8_t* s_gate, float global_gate, const uint8_t* w_up,
                        const uint8_t* s_up, float global_up, const void* x, int64_t ldx,
                        void* y, int64_t ldy, int m, int64_t n, int64_t k, void* workspace,
                        size_t workspace_bytes, uint32_t flags, cudaStream_t stream) {
    bool noop = false;
    int st = check_common(x, ldx, y, ldy, m, n, k, workspace, flags, &noop);
    if (st != NVFP4_OK) return st;
    nvfp4_pro::Prologue pro;
    const Range yr = noop ? Range{0, 0} : rows_range(y, m, ldy, n);
    if ((st = check_pro(prologue, x, ldx, m, k, &yr, noop ? 0 : 1, &pro)) != NVFP4_OK) return st;
    if (noop) return NVFP4_OK;
    if (k > 0) {
        if ((st = check_weight(w_gate, s_gate)) != NVFP4_OK) return st;
        if ((st = check_weight(w_up, s_up)) != NVFP4_OK) return st;
    }
    if ((flags & NVFP4_FLAG_WIDE_TENSOR) && m > NVFP4_PASS_ROWS && k > 0 &&
        pro.kind != NVFP4_PROLOGUE_GATED_RMSNORM && nvfp4_tc::usable(s_gate, k) &&
        nvfp4_tc::usable(s_up, k)) {
        int dev = 0;
        DeviceInfo* di = nullptr;
        if ((st = device_info(&dev, &di)) != NVFP4_OK) return st;
        size_t flags_off, partial_off;
        const size_t base = workspace_layout(di->sms, &flags_off, &partial_off);
        return nvfp4_tc::launch_dual(g_encode, di->sms, w_gate, s_gate, global_gate, w_up, s_up,
                                     global_up, x, ldx, y, ldy, m, n, k, pro, workspace,
                                     workspace_bytes, base, stream);
    }
    if ((st = prologue_pass(pro, &x, &ldx, m, k, workspace, workspace_bytes, flags, stream)) !=
        NVFP4_OK)
        return st;
    const uint8_t* ws_[2] = {w_gate, w_up};
    const uint8_t* ss_[2] = {s_gate, s_up};
    const float gs[2] = {global_gate, global_up};
    return launch<true>(ws_, ss_, gs, x, ldx, y, ldy, m, n, k, workspace, workspace_bytes, flags,
                        stream);
}

int nvfp4_gemv_dual_ex(const uint8_t* w_gate, const uint8_t* s_gate, float global_gate,
                       const uint8_t* w_up, const uint8_t* s_up, float global_up, const void* x,
                       int64_t ldx, void* y, int64_t ldy, int m, int64_t n, int64_t k,
                       void* workspace, size_t workspace_bytes, uint32_t flags,
                       cudaStream_t stream) {
    return nvfp4_gemv_dual_pro(nullptr, w_gate, s_gate, global_gate, w_up, s_up, global_up, x,
                               ldx, y, ldy, m, n, k, workspace, workspace_bytes, flags, stream);
}

int nvfp4_gemv_dual(const uint8_t* w_gate, const uint8_t* s_gate, float global_gate,
                    const uint8_t* w_up, const uint8_t* s_up, float global_up, const void* x,
                    int64_t ldx, void* y, int64_t ldy, int m, int64_t n, int64_t k,
                    void* workspace, size_t workspace_bytes, cudaStream_t stream) {
    return nvfp4_gemv_dual_pro(nullptr, w_gate, s_gate, global_gate, w_up, s_up, global_up, x,
                               ldx, y, ldy, m, n, k, workspace, workspace_bytes, 0u, stream);
}

int nvfp4_gemv_multi_pro(const nvfp4_prologue_t* prologue, const nvfp4_output_t* outputs,
                         int count, const void* x, int64_t ldx, int m, int64_t k,
                         void* workspace, size_t workspace_bytes, uint32_t flags,
                         cudaStream_t stream) {
    if (!outputs) return NVFP4_ERR_NULL;
    if (count < 1 || count > NVFP4_MAX_OUTPUTS) return NVFP4_ERR_SHAPE;
    Span sp[kMaxOutputs];
    Range yr[kMaxOutputs];
    int used = 0;
    for (int o = 0; o < count; ++o) {
        const nvfp4_output_t& a = outputs[o];
        bool noop = false;
        int st = check_common(x, ldx, a.y, a.ldy, m, a.n, k, workspace, flags, &noop);
        if (st != NVFP4_OK) return st;
        if (noop) continue;  // M == 0 or no rows: nothing to write
        if (k > 0 && (st = check_weight(a.w, a.s)) != NVFP4_OK) return st;
        yr[used] = rows_range(a.y, m, a.ldy, a.n);
        Span& b = sp[used++];
        memset(&b, 0, sizeof(b));
        b.w[0] = a.w;
        b.s[0] = a.s;
        b.g[0] = a.global_scale;
        b.y = a.y;
        b.ldy = a.ldy;
        b.n = a.n;
    }
    nvfp4_pro::Prologue pro;
    int st = check_pro(prologue, x, ldx, m, k, yr, used, &pro);
    if (st != NVFP4_OK) return st;
    if (used == 0) return NVFP4_OK;
    int dev = 0;
    DeviceInfo* di = nullptr;
    st = device_info(&dev, &di);
    if (st != NVFP4_OK) return st;
    if ((flags & NVFP4_FLAG_WIDE_TENSOR) && m > NVFP4_PASS_ROWS && k > 0 &&
        pro.kind != NVFP4_PROLOGUE_GATED_RMSNORM) {
        bool all = true;
        for (int o = 0; o < used; ++o) all = all && nvfp4_tc::usable(sp[o].s[0], k);
        if (all) {
            const uint8_t* tw[kMaxOutputs];
            const uint8_t* ts[kMaxOutputs];
            float tg[kMaxOutputs];
            void* ty[kMaxOutputs];
            int64_t tldy[kMaxOutputs], tn[kMaxOutputs];
            for (int o = 0; o < used; ++o) {
                tw[o] = sp[o].w[0];
                ts[o] = sp[o].s[0];
                tg[o] = sp[o].g[0];
                ty[o] = sp[o].y;
                tldy[o] = sp[o].ldy;
                tn[o] = sp[o].n;
            }
            size_t flags_off, partial_off;
            const size_t base = workspace_layout(di->sms, &flags_off, &partial_off);
            return nvfp4_tc::launch_multi(g_encode, di->sms, tw, ts, tg, ty, tldy, tn, used, x,
                                          ldx, m, k, pro, workspace, workspace_bytes, base,
                                          stream);
        }
    }
    if ((st = prologue_pass(pro, &x, &ldx, m, k, workspace, workspace_bytes, flags, stream)) !=
        NVFP4_OK)
        return st;
    using C = Cfg<false>;
    int64_t groups = 0;
    for (int o = 0; o < used; ++o) groups += (sp[o].n + C::kRows - 1) / C::kRows;
    const int64_t cap = max_groups_per_launch<false>(k, di->sms);
    if (used == 1)  // the one-output kernel: bitwise nvfp4_gemv_ex, which also splits its rows
        return launch<false>(sp[0].w, sp[0].s, sp[0].g, x, ldx, sp[0].y, sp[0].ldy, m, sp[0].n,
                             k, workspace, workspace_bytes, flags, stream);
    if (cap < 0 || groups <= cap)
        return launch_spans<false, true>(sp, used, x, ldx, m, k, workspace, workspace_bytes,
                                         flags, stream);
    // too many row groups for one launch at this K: each output as nvfp4_gemv runs it
    for (int o = 0; o < used; ++o) {
        const uint8_t* w_[1] = {sp[o].w[0]};
        const uint8_t* s_[1] = {sp[o].s[0]};
        const float g_[1] = {sp[o].g[0]};
        if ((st = launch<false>(w_, s_, g_, x, ldx, sp[o].y, sp[o].ldy, m, sp[o].n, k, workspace,
                                workspace_bytes, flags, stream)) != NVFP4_OK)
            return st;
    }
    return NVFP4_OK;
}

int nvfp4_gemv_multi(const nvfp4_output_t* outputs, int count, const void* x, int64_t ldx,
                     int m, int64_t k, void* workspace, size_t workspace_bytes, uint32_t flags,
                     cudaStream_t stream) {
    return nvfp4_gemv_multi_pro(nullptr, outputs, count, x, ldx, m, k, workspace,
                                workspace_bytes, flags, stream);
}

int nvfp4_workspace_bytes_wide(int64_t n, int64_t k, int m, size_t* bytes) {
    if (!bytes) return NVFP4_ERR_NULL;
    if (n < 0 || k < 0 || (k % 32) != 0 || k > kMaxK) return NVFP4_ERR_SHAPE;
    if (m < 0 || m > NVFP4_MAX_ROWS) return NVFP4_ERR_ROWS;
    int dev = 0;
    DeviceInfo* di = nullptr;
    int st = device_info(&dev, &di);
    if (st != NVFP4_OK) return st;
    size_t flags_off, partial_off;
    const size_t tier = m > NVFP4_PASS_ROWS ? nvfp4_tc::scratch_bytes(n, k, m, di->sms) : 0;
    const size_t pro = prologue_scratch_bytes(m, k);
    *bytes = workspace_layout(di->sms, &flags_off, &partial_off) + (tier > pro ? tier : pro);
    return NVFP4_OK;
}

int nvfp4_workspace_error(const void* workspace, size_t workspace_bytes, cudaStream_t stream,
                          int32_t* error) {
    if (!error) return NVFP4_ERR_NULL;
    if (!workspace || workspace_bytes < 256 || misaligned(workspace, 16))
        return NVFP4_ERR_WORKSPACE;
    int32_t v = 0;
    if (cudaMemcpyAsync(&v, workspace, sizeof(v), cudaMemcpyDeviceToHost, stream) != cudaSuccess ||
        cudaStreamSynchronize(stream) != cudaSuccess) {
        cudaGetLastError();
        return NVFP4_ERR_LAUNCH;
    }
    *error = v;
    return NVFP4_OK;
}

const char* nvfp4_status_string(int status) {
    switch (status) {
        case NVFP4_OK: return "NVFP4_OK";
        case NVFP4_ERR_NULL: return "NVFP4_ERR_NULL";
        case NVFP4_ERR_SHAPE: return "NVFP4_ERR_SHAPE";
        case NVFP4_ERR_ROWS: return "NVFP4_ERR_ROWS";
        case NVFP4_ERR_ALIGN: return "NVFP4_ERR_ALIGN";
        case NVFP4_ERR_ARCH: return "NVFP4_ERR_ARCH";
        case NVFP4_ERR_LAUNCH: return "NVFP4_ERR_LAUNCH";
        case NVFP4_ERR_WORKSPACE: return "NVFP4_ERR_WORKSPACE";
        case NVFP4_ERR_ALIAS: return "NVFP4_ERR_ALIAS";
        default: return "NVFP4_ERR_UNKNOWN";
    }
}

}  // extern "C"
