// Weight-only NVFP4 GEMV / fused dual GEMV for NVIDIA B200 (sm_100a), with its C ABI.
//
// The operation is the "w4a16_gemv" / "w4a16_gemv_dual" kernel family of a hybrid decoder's
// decode step ("Blueprint - circuit executor" page for qwen3.8-27b-nvfp4 on GB10, table
// "Kernels the plan launches"; weight format "nvfp4/g16", activations bf16, table "Weighted
// nodes"); the fused SiLU(gate)*up epilogue replaces that plan's separate "moe_silu_mul" launch
// (planner setting decode_split_silu).  Row counts 1..8 (8-row speculative draft/verify round,
// kern-qwen38-sm103 model card, section "Run").  Formats and the ABI are described in nvfp4.h.
//
// Design (B200-first):
//   * The path is HBM-bound: 0.5625 bytes per weight.  A persistent grid (a fixed number of
//     CTAs per SM) splits the work -- units of (RB output rows x 128 k) in row-group-major
//     order -- into equal contiguous ranges ("stream-K"), so every SM streams the same number
//     of bytes.  Row groups cut by a range boundary are finished by the CTA holding their first
//     block (the "owner", which reaches them last) after adding the other CTAs' fp32 partials
//     in CTA order; partials and flags live in a caller-provided workspace.  No data atomics:
//     the result is deterministic and the split depends only on (N, K, SM count), never on M.
//   * Each lane streams 16-byte chunks of two weight rows per 16-row tile with L1-bypassing
//     loads, prefetched D units ahead in registers, plus the 2-byte pair of group scales.
//   * Decode in registers with the hardware conversions: cvt e2m1x2 -> f16x2 turns each byte
//     (two nibbles, k and k+1) into an f16 pair, cvt e4m3x2 -> f16x2 turns two scale codes into
//     f16, and one f16x2 multiply gives A = e2m1 * e4m3, exact in f16 (at most 6 significant
//     bits, magnitude in [2^-10, 2688] or zero).
//   * The dot products run on the tensor cores: mma.m16n8k16 (f16 in, fp32 accumulate) with
//     16 weight rows as A and x as B, padded to 8 columns (columns >= M are zero).  The same
//     instruction sequence serves every M, so row m of the output depends only on x row m:
//     bitwise row invariance across M = 1..8.
//   * x is staged once per CTA in shared memory as f16.  Each x row m is scaled by a power of
//     two 2^e(m) chosen from the row's largest magnitude in the CTA's k range (so it lands in
//     [2^14, 2^15)); bf16 values convert exactly unless they are more than 2^31 times smaller
//     than that maximum.  The partial sums are multiplied back by 2^-e(m) (exact) before they
//     are combined.  The scale depends only on row m's data.
//   * Epilogue in fp32: y = acc * g rounded to bf16; the dual computes
//     silu(g_g acc_g) * (g_u acc_u) with expf and rounds once.
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include "nvfp4.h"

namespace {

// ------------------------------------------------------------------------------------------
// geometry

constexpr int kBlockK = 128;         // k per unit (4 lanes x 32)
constexpr int kSlotU4 = 16;          // uint4 of staged f16 x per block per row (256 B)
constexpr int kRowPadU4 = 4;         // 64-byte pad between x rows (bank offset)
constexpr int kMaxRowsPerUnit = 256; // largest RB of any configuration
constexpr int kMaxCtasPerSm = 2;     // largest CTAs/SM of any configuration
constexpr int kPartialFloats = kMaxRowsPerUnit * 8;  // one stream's partial slot
constexpr int kSpinLimit = 1 << 22;  // bounded wait (~0.5-1 s)
constexpr int64_t kMaxK = int64_t(1) << 24;

template <bool DUAL, int WARPS, int R, int D, int MINB>
struct Geo {
    static constexpr int kStreams = DUAL ? 2 : 1;
    static constexpr int kWarps = WARPS;
    static constexpr int kTiles = R;      // 16-row mma tiles per warp
    static constexpr int kDepth = D;      // units prefetched ahead
    static constexpr int kMinBlocks = MINB;
    static constexpr int kThreads = WARPS * 32;
    static constexpr int kRows = WARPS * R * 16;
    static constexpr int kSmemBudget = MINB == 1 ? 200 * 1024 : 100 * 1024;
    static_assert(kRows <= kMaxRowsPerUnit, "unit too tall for the workspace slots");
    static_assert(MINB <= kMaxCtasPerSm, "too many CTAs per SM for the workspace");
};

// Launch configurations (selected at build time; the work split, and therefore the fp32
// summation order, depends on them, never on M).
#ifndef NVFP4_SINGLE_CFG
#define NVFP4_SINGLE_CFG 0
#endif
#ifndef NVFP4_DUAL_CFG
#define NVFP4_DUAL_CFG 0
#endif
#if NVFP4_SINGLE_CFG == 0
using GeoSingle = Geo<false, 8, 2, 3, 1>;
#elif NVFP4_SINGLE_CFG == 1
using GeoSingle = Geo<false, 8, 1, 4, 2>;
#elif NVFP4_SINGLE_CFG == 2
using GeoSingle = Geo<false, 16, 1, 3, 1>;
#else
using GeoSingle = Geo<false, 4, 2, 4, 2>;
#endif
#if NVFP4_DUAL_CFG == 0
using GeoDual = Geo<true, 8, 2, 2, 1>;
#elif NVFP4_DUAL_CFG == 1
using GeoDual = Geo<true, 8, 1, 3, 2>;
#else
using GeoDual = Geo<true, 16, 1, 2, 1>;
#endif

struct Params {
    const uint8_t* w[2];
    const uint8_t* s[2];
    float g[2];          // global scales
    const uint16_t* x;
    int64_t ldx;
    uint16_t* y;
    int64_t ldy;
    int m;
    int64_t n;
    int64_t k;
    int kb;              // 128-k blocks along K (last may be partial)
    int64_t units;       // row groups * kb
    int grid;
    float* partial;      // [grid][2][kPartialFloats]
    uint32_t* flags;     // [grid]
    int32_t* error;
};

// ------------------------------------------------------------------------------------------
// device helpers

__device__ __forceinline__ uint4 ld_stream16(const uint8_t* p) {
    uint4 r;
    asm("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
        : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
        : "l"(p));
    return r;
}

__device__ __forceinline__ uint32_t ld_scale2(const uint8_t* p) {
    unsigned short v;
    asm("ld.global.nc.L1::no_allocate.u16 %0, [%1];" : "=h"(v) : "l"(p));
    return v;
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

__device__ __forceinline__ float bf2f(uint32_t b16) { return __uint_as_float(b16 << 16); }

// One lane's view of one 128-k unit of one weight stream: rows g and g+8 of each tile.
template <int R>
struct UnitRegs {
    uint4 wa[R], wb[R];
    uint32_t sa[R], sb[R];
};

// Per-stream row cursor of a lane: pointers to row (group_row0 + warp*R*16 + g) at k = 32q.
struct RowCursor {
    const uint8_t* w;
    const uint8_t* s;
};

template <int R>
__device__ __forceinline__ void load_unit(UnitRegs<R>& r, const RowCursor& c, uint32_t rows_ok,
                                          bool kok, int b, uint32_t wrow, uint32_t srow) {
#pragma unroll
    for (int t = 0; t < R; ++t) {
        const bool va = kok && ((rows_ok >> (2 * t)) & 1u);
        const bool vb = kok && ((rows_ok >> (2 * t + 1)) & 1u);
        const uint32_t wo = (uint32_t)(16 * t) * wrow + (uint32_t)b * 64u;
        const uint32_t so = (uint32_t)(16 * t) * srow + (uint32_t)b * 8u;
        r.wa[t] = va ? ld_stream16(c.w + wo) : make_uint4(0, 0, 0, 0);
        r.wb[t] = vb ? ld_stream16(c.w + wo + 8u * wrow) : make_uint4(0, 0, 0, 0);
        r.sa[t] = va ? ld_scale2(c.s + so) : 0u;
        r.sb[t] = vb ? ld_scale2(c.s + so + 8u * srow) : 0u;
    }
}

// acc[t][h][i]: tile t, h = 0 for the first mma of each word (k-step A), 1 for the second.
template <int R>
__device__ __forceinline__ void compute_unit(float (&acc)[R][2][4], const UnitRegs<R>& r,
                                             const uint4 (&xv)[4]) {
#pragma unroll
    for (int t = 0; t < R; ++t) {
        const uint32_t Sa = scale_pair(r.sa[t]), Sb = scale_pair(r.sb[t]);
        const uint32_t sa0 = bcast_lo(Sa), sa1 = bcast_hi(Sa);
        const uint32_t sb0 = bcast_lo(Sb), sb1 = bcast_hi(Sb);
        const uint32_t wa[4] = {r.wa[t].x, r.wa[t].y, r.wa[t].z, r.wa[t].w};
        const uint32_t wb[4] = {r.wb[t].x, r.wb[t].y, r.wb[t].z, r.wb[t].w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            uint32_t pa[4], pb[4];
            decode_word(wa[j], pa);
            decode_word(wb[j], pb);
            const uint32_t sA = j < 2 ? sa0 : sa1, sB = j < 2 ? sb0 : sb1;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                pa[i] = hmul2(pa[i], sA);
                pb[i] = hmul2(pb[i], sB);
            }
            // k-step A: logical k {2q, 2q+1 | 2q+8, 2q+9} <- word k {0, 1 | 2, 3}
            mma16816(acc[t][0], pa[0], pb[0], pa[1], pb[1], xv[j].x, xv[j].y);
            // k-step B: word k {4, 5 | 6, 7}
            mma16816(acc[t][1], pa[2], pb[2], pa[3], pb[3], xv[j].z, xv[j].w);
        }
    }
}

// Write this lane's outputs of one tile: c0 (row g, col 2q), c1 (g, 2q+1), c2 (g+8, 2q),
// c3 (g+8, 2q+1).
__device__ __forceinline__ void store_tile(const Params& p, int64_t row0, int g, int q,
                                           const float (&v)[4]) {
    const int64_t ra = row0 + g, rb = ra + 8;
    const int c0 = 2 * q, c1 = 2 * q + 1;
    if (c0 < p.m) {
        if (ra < p.n) p.y[c0 * p.ldy + ra] = f2bf(v[0]);
        if (rb < p.n) p.y[c0 * p.ldy + rb] = f2bf(v[2]);
    }
    if (c1 < p.m) {
        if (ra < p.n) p.y[c1 * p.ldy + ra] = f2bf(v[1]);
        if (rb < p.n) p.y[c1 * p.ldy + rb] = f2bf(v[3]);
    }
}

template <class G>
__device__ __forceinline__ void set_cursor(RowCursor (&c)[2], uint32_t& rows_ok, const Params& p,
                                           int64_t rg, int warp, int g, int q) {
    constexpr int R = G::kTiles;
    const int64_t row = rg * G::kRows + warp * R * 16 + g;
    rows_ok = 0;
#pragma unroll
    for (int t = 0; t < R; ++t) {
        if (row + 16 * t < p.n) rows_ok |= 1u << (2 * t);
        if (row + 16 * t + 8 < p.n) rows_ok |= 1u << (2 * t + 1);
    }
#pragma unroll
    for (int s = 0; s < G::kStreams; ++s) {
        c[s].w = p.w[s] + row * (p.k >> 1) + 16 * q;
        c[s].s = p.s[s] + row * (p.k >> 4) + 2 * q;
    }
}

// ------------------------------------------------------------------------------------------
// the kernel

template <class G>
__global__ void __launch_bounds__(G::kThreads, G::kMinBlocks) nvfp4_gemv_kernel(const Params p) {
    constexpr bool DUAL = G::kStreams == 2;
    constexpr int NS = G::kStreams;
    constexpr int D = G::kDepth;
    constexpr int R = G::kTiles;
    constexpr int NT = G::kThreads;
    extern __shared__ uint4 xsm[];
    __shared__ int s_amax[8];
    __shared__ float s_scale[8], s_descale[8];
    __shared__ int s_ok;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = lane >> 2, q = lane & 3;
    const int cta = blockIdx.x;
    const int64_t U = p.units;
    const int64_t u_begin = U * cta / p.grid;
    const int64_t u_end = U * (cta + 1) / p.grid;
    if (u_begin >= u_end) return;
    const int kb = p.kb;
    const int64_t rg0 = u_begin / kb;
    const int b0 = (int)(u_begin - rg0 * kb);
    const int xslots = (int)((u_end - u_begin) < kb ? (u_end - u_begin) : kb);
    const int xrow = xslots * kSlotU4 + kRowPadU4;  // uint4 per staged x row
    const uint32_t wrow = (uint32_t)(p.k >> 1), srow = (uint32_t)(p.k >> 4);
    const bool last_ok = (int64_t)(kb - 1) * kBlockK + 32 * q < p.k;

    // ---- prefetch the first D units ------------------------------------------------------
    RowCursor pf[2];
    uint32_t pf_rows;
    int64_t pf_rg = rg0;
    int pf_b = b0;
    set_cursor<G>(pf, pf_rows, p, pf_rg, warp, g, q);
    UnitRegs<R> buf[D][NS];
#pragma unroll
    for (int d = 0; d < D; ++d) {
        const bool live = u_begin + d < u_end;
        const bool kok = live && (pf_b != kb - 1 || last_ok);
#pragma unroll
        for (int s = 0; s < NS; ++s) load_unit<R>(buf[d][s], pf[s], pf_rows, kok, pf_b, wrow, srow);
        if (live && ++pf_b == kb) {
            pf_b = 0;
            ++pf_rg;
            set_cursor<G>(pf, pf_rows, p, pf_rg, warp, g, q);
        }
    }

    // ---- stage x as f16, scaled per row by a power of two --------------------------------
    if (tid < 8) s_amax[tid] = 0;
    __syncthreads();
    const int per_row = xslots * kSlotU4;
    for (int mm = 0; mm < p.m; ++mm) {
        float amax = 0.f;
        for (int c = tid; c < per_row; c += NT) {
            const int slot = c >> 4, qq = (c >> 2) & 3, jj = c & 3;
            int blk = b0 + slot;
            if (blk >= kb) blk -= kb;
            const int64_t kk = (int64_t)blk * kBlockK + 32 * qq + 8 * jj;
            if (kk < p.k) {
                const uint4 v = __ldg(reinterpret_cast<const uint4*>(p.x + mm * p.ldx + kk));
                const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    amax = fmaxf(amax, fabsf(bf2f(w4[i] & 0xFFFFu)));
                    amax = fmaxf(amax, fabsf(bf2f(w4[i] >> 16)));
                }
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
        if (lane == 0 && amax > 0.f) atomicMax(&s_amax[mm], __float_as_int(amax));
    }
    __syncthreads();
    if (tid < 8) {
        // amax in [2^E, 2^(E+1)) -> scale 2^(14-E) puts it in [2^14, 2^15), inside f16's range
        const uint32_t bits = (uint32_t)s_amax[tid];
        int e = 0;
        const int E = (int)((bits >> 23) & 0xFF) - 127;
        if (bits != 0 && E < 128) e = 14 - E;
        e = e > 126 ? 126 : (e < -126 ? -126 : e);
        s_scale[tid] = __uint_as_float((uint32_t)(e + 127) << 23);
        s_descale[tid] = __uint_as_float((uint32_t)(127 - e) << 23);
    }
    __syncthreads();
    for (int mm = 0; mm < p.m; ++mm) {
        const float sc = s_scale[mm];
        for (int c = tid; c < per_row; c += NT) {
            const int slot = c >> 4, qq = (c >> 2) & 3, jj = c & 3;
            int blk = b0 + slot;
            if (blk >= kb) blk -= kb;
            const int64_t kk = (int64_t)blk * kBlockK + 32 * qq + 8 * jj;
            uint4 o = make_uint4(0, 0, 0, 0);
            if (kk < p.k) {
                const uint4 v = __ldg(reinterpret_cast<const uint4*>(p.x + mm * p.ldx + kk));
                const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
                uint32_t h[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const __half2 t = __floats2half2_rn(bf2f(w4[i] & 0xFFFFu) * sc,
                                                        bf2f(w4[i] >> 16) * sc);
                    h[i] = *reinterpret_cast<const uint32_t*>(&t);
                }
                o = make_uint4(h[0], h[1], h[2], h[3]);
            }
            // swizzle the 16-byte chunk so the 4 lanes of a row hit distinct banks
            xsm[mm * xrow + slot * kSlotU4 + qq * 4 + (jj ^ qq)] = o;
        }
    }
    __syncthreads();
    const float ds0 = 2 * q < p.m ? s_descale[2 * q] : 1.f;
    const float ds1 = 2 * q + 1 < p.m ? s_descale[2 * q + 1] : 1.f;

    float acc[NS][R][2][4];
#pragma unroll
    for (int s = 0; s < NS; ++s)
#pragma unroll
        for (int t = 0; t < R; ++t)
#pragma unroll
            for (int h = 0; h < 2; ++h)
#pragma unroll
                for (int i = 0; i < 4; ++i) acc[s][t][h][i] = 0.f;

    float* const my_partial = p.partial + (int64_t)cta * 2 * kPartialFloats;
    int64_t u = u_begin;
    int64_t cur_rg = rg0;
    int cur_b = b0, seg_b0 = b0;

    while (u < u_end) {
#pragma unroll
        for (int d = 0; d < D; ++d) {
            if (u >= u_end) break;
            UnitRegs<R> cur[NS];
            {
                const bool live = u + D < u_end;
                const bool kok = live && (pf_b != kb - 1 || last_ok);
#pragma unroll
                for (int s = 0; s < NS; ++s) {
                    cur[s] = buf[d][s];
                    load_unit<R>(buf[d][s], pf[s], pf_rows, kok, pf_b, wrow, srow);
                }
                if (live && ++pf_b == kb) {
                    pf_b = 0;
                    ++pf_rg;
                    set_cursor<G>(pf, pf_rows, p, pf_rg, warp, g, q);
                }
            }
            int slot = cur_b - b0;
            if (slot < 0) slot += kb;
            uint4 xv[4];
#pragma unroll
            for (int j = 0; j < 4; ++j)
                xv[j] = g < p.m ? xsm[g * xrow + slot * kSlotU4 + q * 4 + (j ^ q)]
                                : make_uint4(0, 0, 0, 0);
#pragma unroll
            for (int s = 0; s < NS; ++s) compute_unit<R>(acc[s], cur[s], xv);
            ++u;

            if (cur_b + 1 == kb || u == u_end) {
                // ---- end of a row-group segment: blocks seg_b0 .. cur_b of row group cur_rg
                float tot[2][R][4];
#pragma unroll
                for (int s = 0; s < NS; ++s)
#pragma unroll
                    for (int t = 0; t < R; ++t)
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            tot[s][t][i] = (acc[s][t][0][i] + acc[s][t][1][i]) * ((i & 1) ? ds1 : ds0);
                            acc[s][t][0][i] = 0.f;
                            acc[s][t][1][i] = 0.f;
                        }
                if (seg_b0 > 0) {
                    // contributor: the row group started before this CTA's range
                    if (2 * q < p.m) {
#pragma unroll
                        for (int s = 0; s < NS; ++s)
#pragma unroll
                            for (int t = 0; t < R; ++t) {
                                float* dst = my_partial + s * kPartialFloats +
                                             ((warp * R + t) * 32 + lane) * 4;
                                *reinterpret_cast<float4*>(dst) = make_float4(
                                    tot[s][t][0], tot[s][t][1], tot[s][t][2], tot[s][t][3]);
                            }
                    }
                    __threadfence();
                    __syncthreads();
                    if (tid == 0) st_release(p.flags + cta, 1u);
                } else {
                    if (cur_b + 1 != kb) {
                        // owner: the following CTAs hold the rest of this row group, each as
                        // the first segment of its range; add their partials in CTA order
                        for (int c2 = cta + 1; c2 < p.grid; ++c2) {
                            if (U * c2 / p.grid >= (cur_rg + 1) * kb) break;
                            if (tid == 0) {
                                int it = 0;
                                while (ld_acquire(p.flags + c2) == 0u && ++it < kSpinLimit)
                                    __nanosleep(32);
                                s_ok = it < kSpinLimit;
                                if (s_ok) p.flags[c2] = 0u;
                                else atomicExch(p.error, 1);
                            }
                            __syncthreads();
                            if (s_ok && 2 * q < p.m) {
                                const float* src = p.partial + (int64_t)c2 * 2 * kPartialFloats;
#pragma unroll
                                for (int s = 0; s < NS; ++s)
#pragma unroll
                                    for (int t = 0; t < R; ++t) {
                                        const float4 v = ld_cg4(src + s * kPartialFloats +
                                                                ((warp * R + t) * 32 + lane) * 4);
                                        tot[s][t][0] += v.x;
                                        tot[s][t][1] += v.y;
                                        tot[s][t][2] += v.z;
                                        tot[s][t][3] += v.w;
                                    }
                            }
                            __syncthreads();
                        }
                    }
#pragma unroll
                    for (int t = 0; t < R; ++t) {
                        const int64_t row0 = cur_rg * G::kRows + (warp * R + t) * 16;
                        float v[4];
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            if (DUAL) {
                                const float a = tot[0][t][i] * p.g[0];
                                const float b = tot[1][t][i] * p.g[1];
                                v[i] = a / (1.0f + expf(-a)) * b;
                            } else {
                                v[i] = tot[0][t][i] * p.g[0];
                            }
                        }
                        store_tile(p, row0, g, q, v);
                    }
                }
                seg_b0 = 0;
            }
            if (++cur_b == kb) {
                cur_b = 0;
                ++cur_rg;
            }
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
bool g_attr_set[2][64];

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
    *dev_out = dev;
    *info = &di;
    return NVFP4_OK;
}

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// workspace: [error int32 | pad to 256][flags uint32[ctas] | pad to 256][partials]
size_t workspace_layout(int sms, size_t* flags_off, size_t* partial_off) {
    const size_t ctas = (size_t)sms * kMaxCtasPerSm;
    *flags_off = 256;
    *partial_off = 256 + align_up(ctas * 4, 256);
    return *partial_off + ctas * 2 * kPartialFloats * sizeof(float);
}

bool misaligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) != 0; }

int check_common(const void* x, int64_t ldx, const void* y, int64_t ldy, int m, int64_t n,
                 int64_t k, const void* ws, bool* noop) {
    *noop = false;
    if (m < 0 || m > NVFP4_MAX_ROWS) return NVFP4_ERR_ROWS;
    if (n < 0 || k < 0 || (k % 32) != 0 || k > kMaxK) return NVFP4_ERR_SHAPE;
    if (m == 0 || n == 0) {
        *noop = true;
        return NVFP4_OK;
    }
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

template <class G>
int launch(const uint8_t* const* w, const uint8_t* const* s, const float* gs, const void* x,
           int64_t ldx, void* y, int64_t ldy, int m, int64_t n, int64_t k, void* ws,
           size_t ws_bytes, cudaStream_t stream) {
    constexpr bool DUAL = G::kStreams == 2;
    int dev = 0;
    DeviceInfo* di = nullptr;
    int st = device_info(&dev, &di);
    if (st != NVFP4_OK) return st;
    size_t flags_off, partial_off;
    const size_t need = workspace_layout(di->sms, &flags_off, &partial_off);
    if (ws_bytes < need) return NVFP4_ERR_WORKSPACE;

    if (k == 0) {  // empty sum: y = 0 (silu(0) * 0 = 0 for the dual)
        if (cudaMemset2DAsync(y, (size_t)ldy * 2, 0, (size_t)n * 2, (size_t)m, stream) !=
            cudaSuccess) {
            cudaGetLastError();
            return NVFP4_ERR_LAUNCH;
        }
        return NVFP4_OK;
    }

    if (!g_attr_set[DUAL][dev]) {
        if (cudaFuncSetAttribute(nvfp4_gemv_kernel<G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 G::kSmemBudget) != cudaSuccess) {
            cudaGetLastError();
            return NVFP4_ERR_LAUNCH;
        }
        g_attr_set[DUAL][dev] = true;
    }

    const int kb = (int)((k + kBlockK - 1) / kBlockK);
    const size_t slot_bytes = (size_t)kSlotU4 * 16;  // 256 B of staged x per block per row
    const int max_grid = di->sms * G::kMinBlocks;
    // Rows per launch: the staged x (M rows x blocks of a CTA's range) must fit the shared
    // memory budget; a range spans at most ceil(units / grid) blocks, capped at kb.  Sized for
    // the largest M so that the work split never depends on M.
    int64_t rows_per_launch = n;
    {
        const size_t mx = NVFP4_MAX_ROWS;
        const int64_t max_slots =
            (int64_t)((G::kSmemBudget - mx * kRowPadU4 * 16) / (mx * slot_bytes));
        if (max_slots < kb) {
            const int64_t groups = (int64_t)max_grid * max_slots / kb;
            const int64_t cap = (groups > 0 ? groups : 1) * G::kRows;
            if (cap < rows_per_launch) rows_per_launch = cap;
        }
    }

    char* wsb = static_cast<char*>(ws);
    for (int64_t r0 = 0; r0 < n; r0 += rows_per_launch) {
        const int64_t nn = (n - r0) < rows_per_launch ? (n - r0) : rows_per_launch;
        Params p;
        for (int i = 0; i < 2; ++i) {
            const int src = DUAL ? i : 0;
            p.w[i] = w[src] + r0 * (k / 2);
            p.s[i] = s[src] + r0 * (k / 16);
            p.g[i] = gs[src];
        }
        p.x = static_cast<const uint16_t*>(x);
        p.ldx = ldx;
        p.y = static_cast<uint16_t*>(y) + r0;
        p.ldy = ldy;
        p.m = m;
        p.n = nn;
        p.k = k;
        p.kb = kb;
        p.units = ((nn + G::kRows - 1) / G::kRows) * kb;
        p.grid = (int)(p.units < max_grid ? p.units : max_grid);
        p.partial = reinterpret_cast<float*>(wsb + partial_off);
        p.flags = reinterpret_cast<uint32_t*>(wsb + flags_off);
        p.error = reinterpret_cast<int32_t*>(wsb);
        const int64_t max_range = (p.units + p.grid - 1) / p.grid;
        const int slots = (int)(max_range < kb ? max_range : kb);
        const size_t smem = (size_t)m * ((size_t)slots * slot_bytes + kRowPadU4 * 16);
        nvfp4_gemv_kernel<G><<<p.grid, G::kThreads, smem, stream>>>(p);
        if (cudaGetLastError() != cudaSuccess) return NVFP4_ERR_LAUNCH;
    }
    return NVFP4_OK;
}

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

int nvfp4_gemv(const uint8_t* w, const uint8_t* s, float global_scale, const void* x,
               int64_t ldx, void* y, int64_t ldy, int m, int64_t n, int64_t k, void* workspace,
               size_t workspace_bytes, cudaStream_t stream) {
    bool noop = false;
    int st = check_common(x, ldx, y, ldy, m, n, k, workspace, &noop);
    if (st != NVFP4_OK || noop) return st;
    if (k > 0 && (st = check_weight(w, s)) != NVFP4_OK) return st;
    const uint8_t* ws_[1] = {w};
    const uint8_t* ss_[1] = {s};
    const float gs[1] = {global_scale};
    return launch<GeoSingle>(ws_, ss_, gs, x, ldx, y, ldy, m, n, k, workspace, workspace_bytes,
                             stream);
}

int nvfp4_gemv_dual(const uint8_t* w_gate, const uint8_t* s_gate, float global_gate,
                    const uint8_t* w_up, const uint8_t* s_up, float global_up, const void* x,
                    int64_t ldx, void* y, int64_t ldy, int m, int64_t n, int64_t k,
                    void* workspace, size_t workspace_bytes, cudaStream_t stream) {
    bool noop = false;
    int st = check_common(x, ldx, y, ldy, m, n, k, workspace, &noop);
    if (st != NVFP4_OK || noop) return st;
    if (k > 0) {
        if ((st = check_weight(w_gate, s_gate)) != NVFP4_OK) return st;
        if ((st = check_weight(w_up, s_up)) != NVFP4_OK) return st;
    }
    const uint8_t* ws_[2] = {w_gate, w_up};
    const uint8_t* ss_[2] = {s_gate, s_up};
    const float gs[2] = {global_gate, global_up};
    return launch<GeoDual>(ws_, ss_, gs, x, ldx, y, ldy, m, n, k, workspace, workspace_bytes,
                           stream);
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
        default: return "NVFP4_ERR_UNKNOWN";
    }
}

}  // extern "C"
