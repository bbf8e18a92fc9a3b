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
//   * The path is HBM-bound: 0.5625 bytes per weight.  A persistent grid (one CTA per SM)
//     splits the work -- units of (256 output rows x 128 k) in row-group-major order -- into
//     equal contiguous ranges ("stream-K"), so every SM streams the same number of bytes.
//     Row groups cut by a range boundary are finished by the CTA holding their first block
//     (the "owner", which reaches them last) after adding the other CTAs' fp32 partials in
//     CTA order; partials and flags live in a caller-provided workspace.  No data atomics:
//     the result is deterministic and the split depends only on (N, K, SM count), never on M.
//   * Each lane streams 16-byte chunks of two weight rows with L1-bypassing loads, prefetched
//     DEPTH units ahead in registers, plus the 2-byte pair of group scales that covers them.
//   * Decode in registers, exact: an e2m1 nibble is placed into the exponent/mantissa bits of
//     a bf16 (value * 2^-126, subnormal for 0.5), two nibbles 16 bits apart per bf16x2 word;
//     the group scale comes from cvt e4m3x2 -> f16x2, re-based to bf16 (s * 2^119) by bit moves
//     and two bf16x2 multiplies; one bf16x2 multiply then gives A = e2m1 * e4m3 * 2^-7, which
//     is exact in bf16 (at most 6 significant bits, range 2^-17 .. 21).
//   * The dot products run on the tensor cores: mma.m16n8k16 (bf16 in, fp32 accumulate) with
//     16 weight rows as A and x as B, padded to 8 columns (columns >= M are zero).  The same
//     instruction sequence serves every M, so row m of the output depends only on x row m:
//     bitwise row invariance across M = 1..8.  The k order inside an mma is a permutation of
//     physical k chosen so that each lane's decoded words feed A directly; x is staged in
//     shared memory once per CTA already permuted to match.
//   * Epilogue in fp32: y = acc * (g * 2^7) rounded to bf16; the dual computes
//     silu(g_g acc_g) * (g_u acc_u) with expf and rounds once.
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include "nvfp4.h"

namespace {

// ------------------------------------------------------------------------------------------
// geometry

constexpr int kWarps = 8;                                   // warps per CTA
constexpr int kTilesPerWarp = 2;                            // 16-row mma tiles per warp
constexpr int kThreads = kWarps * 32;
constexpr int kRowsPerGroup = kWarps * kTilesPerWarp * 16;  // 256 output rows per unit
constexpr int kBlockK = 128;                                // k per unit (4 lanes x 32)
constexpr int kSlotU4 = 16;                                 // uint4 per staged x block per row
constexpr int kRowPadU4 = 4;                                // 64-byte pad between x rows
constexpr int kSmemBudget = 200 * 1024;
constexpr int kPartialFloats = kRowsPerGroup * 8;           // one stream's partial (16 KB / 2)
constexpr int kSpinLimit = 1 << 22;                         // bounded wait (~0.5-1 s)

template <bool DUAL>
struct Cfg {
    static constexpr int kStreams = DUAL ? 2 : 1;
    static constexpr int kDepth = DUAL ? 2 : 4;  // units prefetched ahead
};

struct Params {
    const uint8_t* w[2];
    const uint8_t* s[2];
    float geff[2];       // global scale * 2^7
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

__device__ __forceinline__ uint32_t bmul2(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// Two e4m3 scale codes (low byte = even group, high byte = odd group) -> bf16x2 of s * 2^119.
// cvt gives f16 s exactly (every e4m3 value is a normal f16 or zero); shifting the f16 bits
// right by 3 re-reads them as a bf16 of value s * 2^-112 (same exponent field, bf16 keeps the
// top 7 of f16's 10 mantissa bits, and e4m3 uses only 3).  Two exact multiplies by 2^116 and
// 2^115 bring it to s * 2^119 (at most 1.75 * 2^127, inside bf16's range).
__device__ __forceinline__ uint32_t scale_pair(uint32_t codes) {
    uint32_t h;
    asm("{\n\t.reg .b16 t;\n\tcvt.u16.u32 t, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, t;\n\t}"
        : "=r"(h)
        : "r"(codes));
    uint32_t t = (h >> 3) & 0x0FFF0FFFu;
    t = bmul2(t, 0x79807980u);     // 2^116
    return bmul2(t, 0x79007900u);  // 2^115
}

__device__ __forceinline__ uint32_t bcast_lo(uint32_t v) { return __byte_perm(v, 0, 0x1010); }
__device__ __forceinline__ uint32_t bcast_hi(uint32_t v) { return __byte_perm(v, 0, 0x3232); }

// 8 e2m1 nibbles (k = 0..7 of a word, nibble i in bits 4i..4i+3) -> 4 bf16x2 words
// p[i] = {lo: nibble i, hi: nibble i+4}, each of value e2m1 * 2^-126 (bits: sign at 15,
// exponent field = e2m1 exponent, mantissa msb = e2m1 mantissa).
__device__ __forceinline__ void decode_word(uint32_t w, uint32_t (&p)[4]) {
    const uint32_t MAG = 0x01C001C0u, SGN = 0x80008000u;
    p[0] = ((w << 6) & MAG) | ((w << 12) & SGN);
    p[1] = ((w << 2) & MAG) | ((w << 8) & SGN);
    p[2] = ((w >> 2) & MAG) | ((w << 4) & SGN);
    p[3] = ((w >> 6) & MAG) | (w & SGN);
}

__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
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

// One lane's view of one 128-k unit of one weight stream: rows g and g+8 of each tile.
template <int R>
struct UnitRegs {
    uint4 wa[R], wb[R];
    uint32_t sa[R], sb[R];
};

template <int R>
__device__ __forceinline__ void load_unit(UnitRegs<R>& r, const uint8_t* w, const uint8_t* s,
                                          const Params& p, int64_t u, int warp, int g, int q,
                                          bool live) {
    const int64_t rg = u / p.kb;
    const int b = (int)(u - rg * p.kb);
    const bool kvalid = live && ((int64_t)b * kBlockK + 32 * q < p.k);
    const int64_t wrow = p.k >> 1, srow = p.k >> 4;
#pragma unroll
    for (int t = 0; t < R; ++t) {
        const int64_t ra = rg * kRowsPerGroup + (warp * R + t) * 16 + g;
        const int64_t rb = ra + 8;
        const bool va = kvalid && ra < p.n, vb = kvalid && rb < p.n;
        const int64_t wo = (int64_t)b * 64 + 16 * q, so = (int64_t)b * 8 + 2 * q;
        r.wa[t] = va ? ld_stream16(w + ra * wrow + wo) : make_uint4(0, 0, 0, 0);
        r.wb[t] = vb ? ld_stream16(w + rb * wrow + wo) : make_uint4(0, 0, 0, 0);
        r.sa[t] = va ? ld_scale2(s + ra * srow + so) : 0u;
        r.sb[t] = vb ? ld_scale2(s + rb * srow + so) : 0u;
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
                pa[i] = bmul2(pa[i], sA);
                pb[i] = bmul2(pb[i], sB);
            }
            // k-step A: logical k {2q, 2q+1, 2q+8, 2q+9} <- nibbles {0, 4, 1, 5} of the word
            mma16816(acc[t][0], pa[0], pb[0], pa[1], pb[1], xv[j].x, xv[j].y);
            // k-step B: nibbles {2, 6, 3, 7}
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

template <bool DUAL, int R>
__device__ __forceinline__ void epilogue(const Params& p, const float (&tot)[2][R][4], int64_t rg,
                                         int warp, int g, int q) {
#pragma unroll
    for (int t = 0; t < R; ++t) {
        const int64_t row0 = rg * kRowsPerGroup + (warp * R + t) * 16;
        float v[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            if (DUAL) {
                const float a = tot[0][t][i] * p.geff[0];
                const float b = tot[1][t][i] * p.geff[1];
                v[i] = a / (1.0f + expf(-a)) * b;
            } else {
                v[i] = tot[0][t][i] * p.geff[0];
            }
        }
        store_tile(p, row0, g, q, v);
    }
}

// ------------------------------------------------------------------------------------------
// the kernel

template <bool DUAL>
__global__ void __launch_bounds__(kThreads, 1) nvfp4_gemv_kernel(const Params p) {
    constexpr int NS = Cfg<DUAL>::kStreams;
    constexpr int D = Cfg<DUAL>::kDepth;
    constexpr int R = kTilesPerWarp;
    extern __shared__ uint4 xsm[];

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = lane >> 2, q = lane & 3;
    const int cta = blockIdx.x;
    const int64_t U = p.units;
    const int64_t u_begin = U * cta / p.grid;
    const int64_t u_end = U * (cta + 1) / p.grid;
    if (u_begin >= u_end) return;
    const int kb = p.kb;
    const int b0 = (int)(u_begin % kb);
    const int xslots = (int)((u_end - u_begin) < kb ? (u_end - u_begin) : kb);
    const int xrow = xslots * kSlotU4 + kRowPadU4;  // uint4 per staged x row

    // prefetch the first D units before staging x
    UnitRegs<R> buf[D][NS];
#pragma unroll
    for (int d = 0; d < D; ++d)
#pragma unroll
        for (int s = 0; s < NS; ++s)
            load_unit<R>(buf[d][s], p.w[s], p.s[s], p, u_begin + d, warp, g, q,
                         u_begin + d < u_end);

    // stage x for blocks b0 .. b0+xslots-1 (mod kb), permuted to the mma B-fragment order:
    // xsm[m][slot][j][q] = {x0,x4},{x1,x5},{x2,x6},{x3,x7} of k = blk*128 + 32q + 8j + 0..7
    const int total = p.m * xslots * kSlotU4;
    for (int i = tid; i < total; i += kThreads) {
        const int qq = i & 3, jj = (i >> 2) & 3;
        const int slot = (i >> 4) % xslots, mm = (i >> 4) / xslots;
        int blk = b0 + slot;
        if (blk >= kb) blk -= kb;
        const int64_t kk = (int64_t)blk * kBlockK + 32 * qq + 8 * jj;
        uint4 o = make_uint4(0, 0, 0, 0);
        if (kk < p.k) {
            const uint4 v = *reinterpret_cast<const uint4*>(p.x + mm * p.ldx + kk);
            o.x = __byte_perm(v.x, v.z, 0x5410);
            o.y = __byte_perm(v.x, v.z, 0x7632);
            o.z = __byte_perm(v.y, v.w, 0x5410);
            o.w = __byte_perm(v.y, v.w, 0x7632);
        }
        xsm[mm * xrow + slot * kSlotU4 + jj * 4 + qq] = o;
    }
    __syncthreads();

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

    for (int64_t base = u_begin; base < u_end; base += D) {
#pragma unroll
        for (int d = 0; d < D; ++d) {
            const int64_t u = base + d;
            if (u >= u_end) break;
            UnitRegs<R> cur[NS];
#pragma unroll
            for (int s = 0; s < NS; ++s) {
                cur[s] = buf[d][s];
                load_unit<R>(buf[d][s], p.w[s], p.s[s], p, u + D, warp, g, q, u + D < u_end);
            }
            const int64_t rg = u / kb;
            const int b = (int)(u - rg * kb);
            int slot = b - b0;
            if (slot < 0) slot += kb;
            uint4 xv[4];
#pragma unroll
            for (int j = 0; j < 4; ++j)
                xv[j] = g < p.m ? xsm[g * xrow + slot * kSlotU4 + j * 4 + q]
                                : make_uint4(0, 0, 0, 0);
#pragma unroll
            for (int s = 0; s < NS; ++s) compute_unit<R>(acc[s], cur[s], xv);

            if (b + 1 != kb && u + 1 != u_end) continue;

            // ---- end of a row-group segment -------------------------------------------
            const int64_t seg_first = u_begin > rg * kb ? u_begin : rg * kb;
            const int seg_b0 = (int)(seg_first - rg * kb);
            float tot[2][R][4];
#pragma unroll
            for (int s = 0; s < NS; ++s)
#pragma unroll
                for (int t = 0; t < R; ++t)
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        tot[s][t][i] = acc[s][t][0][i] + acc[s][t][1][i];
                        acc[s][t][0][i] = 0.f;
                        acc[s][t][1][i] = 0.f;
                    }
            if (seg_b0 > 0) {
                // contributor: this CTA's first segment starts inside the row group
                if (2 * q < p.m) {
#pragma unroll
                    for (int s = 0; s < NS; ++s)
#pragma unroll
                        for (int t = 0; t < R; ++t) {
                            float* dst = my_partial + s * kPartialFloats +
                                         ((warp * R + t) * 32 + lane) * 4;
                            *reinterpret_cast<float4*>(dst) =
                                make_float4(tot[s][t][0], tot[s][t][1], tot[s][t][2],
                                            tot[s][t][3]);
                        }
                }
                __threadfence();
                __syncthreads();
                if (tid == 0) st_release(p.flags + cta, 1u);
                continue;
            }
            if (b + 1 != kb) {
                // owner: this segment starts at the row group's first block and ends before
                // its last; the following CTAs hold the rest, each as its first segment.
                for (int c2 = cta + 1; c2 < p.grid; ++c2) {
                    const int64_t ub2 = U * c2 / p.grid;
                    if (ub2 >= (rg + 1) * kb) break;
                    __shared__ int ok;
                    if (tid == 0) {
                        int it = 0;
                        while (ld_acquire(p.flags + c2) == 0u && ++it < kSpinLimit)
                            __nanosleep(64);
                        ok = it < kSpinLimit;
                        if (ok) p.flags[c2] = 0u;
                        else atomicExch(p.error, 1);
                    }
                    __syncthreads();
                    if (ok && 2 * q < p.m) {
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
            epilogue<DUAL, R>(p, tot, rg, warp, g, q);
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

// workspace: [error int32 | pad to 256][flags uint32[sms] | pad to 256][partials]
size_t workspace_layout(int sms, size_t* flags_off, size_t* partial_off) {
    *flags_off = 256;
    *partial_off = 256 + align_up((size_t)sms * 4, 256);
    return *partial_off + (size_t)sms * 2 * kPartialFloats * sizeof(float);
}

bool misaligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) != 0; }

int check_common(const void* x, int64_t ldx, const void* y, int64_t ldy, int m, int64_t n,
                 int64_t k, const void* ws, bool* noop) {
    *noop = false;
    if (m < 0 || m > NVFP4_MAX_ROWS) return NVFP4_ERR_ROWS;
    if (n < 0 || k < 0 || (k % 32) != 0 || k > (int64_t(1) << 30)) return NVFP4_ERR_SHAPE;
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

template <bool DUAL>
int launch(const uint8_t* const* w, const uint8_t* const* s, const float* gs, const void* x,
           int64_t ldx, void* y, int64_t ldy, int m, int64_t n, int64_t k, void* ws,
           size_t ws_bytes, cudaStream_t stream) {
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
        if (cudaFuncSetAttribute(nvfp4_gemv_kernel<DUAL>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 kSmemBudget) != cudaSuccess) {
            cudaGetLastError();
            return NVFP4_ERR_LAUNCH;
        }
        g_attr_set[DUAL][dev] = true;
    }

    const int kb = (int)((k + kBlockK - 1) / kBlockK);
    const size_t bytes_per_slot_row = (size_t)kSlotU4 * 16;  // 256 B of x per block per row
    // Rows per launch: the staged x (M rows x blocks of the CTA's range) must fit the shared
    // memory budget.  A CTA's range spans at most ceil(units / grid) blocks, capped at kb.
    // Sized for the largest M so that the work split never depends on M.
    int64_t rows_per_launch = n;
    {
        const size_t mx = NVFP4_MAX_ROWS;
        const int64_t max_slots =
            (int64_t)((kSmemBudget - mx * kRowPadU4 * 16) / (mx * bytes_per_slot_row));
        if (max_slots < kb) {
            // need ceil(ceil(rows/256)*kb / sms) <= max_slots
            const int64_t groups = (int64_t)di->sms * max_slots / kb;
            const int64_t cap = (groups > 0 ? groups : 1) * kRowsPerGroup;
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
            p.geff[i] = gs[src] * 128.0f;
        }
        p.x = static_cast<const uint16_t*>(x);
        p.ldx = ldx;
        p.y = static_cast<uint16_t*>(y) + r0;
        p.ldy = ldy;
        p.m = m;
        p.n = nn;
        p.k = k;
        p.kb = kb;
        p.units = ((nn + kRowsPerGroup - 1) / kRowsPerGroup) * kb;
        p.grid = (int)(p.units < di->sms ? p.units : di->sms);
        p.partial = reinterpret_cast<float*>(wsb + partial_off);
        p.flags = reinterpret_cast<uint32_t*>(wsb + flags_off);
        p.error = reinterpret_cast<int32_t*>(wsb);
        const int64_t max_range = (p.units + p.grid - 1) / p.grid;
        const int slots = (int)(max_range < kb ? max_range : kb);
        const size_t smem = (size_t)m * ((size_t)slots * bytes_per_slot_row + kRowPadU4 * 16);
        nvfp4_gemv_kernel<DUAL><<<p.grid, kThreads, smem, stream>>>(p);
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
    return launch<false>(ws_, ss_, gs, x, ldx, y, ldy, m, n, k, workspace, workspace_bytes,
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
    return launch<true>(ws_, ss_, gs, x, ldx, y, ldy, m, n, k, workspace, workspace_bytes,
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
