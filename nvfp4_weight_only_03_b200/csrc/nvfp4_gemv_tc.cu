// Tensor-core tier of the NVFP4 GEMV for calls of more than 8 rows (NVFP4_FLAG_WIDE_TENSOR):
// the plan's wider multi_seq arms of up to 128 rows ("Blueprint - circuit executor" page for
// qwen3.8-27b-nvfp4 on GB10, table "Plan arms"; planner setting w4a16_tc=on).  From about 32
// rows the contraction outgrows the warp-level mma of the 1..8-row kernel, so this tier uses
// the 5th-generation tensor cores: tcgen05.mma kind::f16 with f16 operands (A the decoded
// weights, B the f16 copy of x), fp32 accumulators in tensor memory.
//
//   D[n][m] = sum_k W(n, k) * x'[m][k]    (128 weight rows n of a tile by N x rows m)
//
// * x': nvfp4_tc_prep writes an f16 copy of x to the workspace (after the call's prologue, if
//   any), row m scaled by the power of two 2^e(m) that puts its largest magnitude in
//   [2^14, 2^15), and the row's descale 2^-e(m); the epilogues multiply by it.
// * Work: a tile is 128 weight rows; K is cut into `splits` equal ranges of 256-k units, and
//   each CTA (two per SM) computes one (tile, split) item.  The split depends only on (N, K,
//   SM count).  With one split the CTA writes y; otherwise it writes fp32 partials to the
//   workspace and nvfp4_tc_reduce adds the splits in order (the dual: nvfp4_tc_dual_finish,
//   over both streams).  Deterministic, no atomics.
// * A producer warp loads with TMA (no multicast), per 256-k unit the 128 weight rows' packed
//   nibbles (128 bytes each, 128-byte swizzle) and scale codes, and per 64-k stage the x' tile
//   (N rows x 64 k of f16, 128-byte swizzle: the MMA's K-major B layout; rows >= M read as zero).
// * Eight decode warps (two threads per weight row) turn each stage's nibbles into f16 weights:
//   cvt e2m1x2 -> f16x2 times the e4m3 scale in f16 (exact: at most 6 significant bits), stored
//   as the MMA's K-major A tile (128-byte swizzle) in one of NVFP4_TC_ABUF buffers.
// * One MMA thread issues 4 x tcgen05.mma (M = 128, N = M rounded up to 16, K = 16) per stage
//   into one fp32 accumulator of up to 128 tensor-memory columns, and frees the stage and the A
//   buffer with tcgen05.commit.  Four warps then read the accumulator (tcgen05.ld) and write out.
// * Every x row is computed by the same instructions whatever M is (the MMA's columns do not
//   depend on each other), so rows are bitwise invariant for every M in 9..128.  Against calls of
//   1..8 rows (a different instruction sequence and a different x scaling) rows agree within the
//   tolerance.
// * Waits are bounded: a wait that gives up records an error in the workspace's error word,
//   and tensor memory is freed on every path.
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include "nvfp4.h"
#include "nvfp4_tc.h"

namespace {

constexpr int kRows = 128;                  // weight rows per tile (MMA M)
constexpr int kMaxXRows = 128;              // x rows per MMA at most (MMA N)
constexpr int kStageK = 64;                 // k per stage
constexpr int kUnitK = 256;                 // k per scale box (16 codes per row)
constexpr int kXRowBytes = kStageK * 2;     // 128: one x row of a stage, f16
constexpr int kWBytes = kRows * kUnitK / 2;     // 16384: a unit's packed nibbles, 128 B per row
constexpr int kSBytes = kRows * 16;             // 2048: the unit's scale codes
constexpr int kUnitBytes = kWBytes + kSBytes;   // 18432 = 18 x 1024
constexpr int kSub = kUnitK / kStageK;          // 4 stages per unit
constexpr int kABytes = kRows * kStageK * 2;    // 16384: decoded f16 tile
#ifndef NVFP4_TC_ABUF
#define NVFP4_TC_ABUF 2
#endif
constexpr int kStages = 6;                  // x tiles in flight at most (one per 64-k stage)
constexpr int kUStages = 2;                 // weight units in flight (one per 256 k)
// Two CTAs share an SM: each CTA's stages are bound by its own hand-offs (TMA -> decode -> MMA
// -> commit), not by a resource the SM's other CTA needs, so a second CTA overlaps them.  Each
// then has half of the SM's shared memory (228 KB, less 1 KB reserved per CTA).
constexpr int kCtasPerSm = 2;
constexpr size_t kCtaSmemBudget = 233472 / kCtasPerSm - 1024;
constexpr int kABuf = NVFP4_TC_ABUF;        // decoded tiles in flight
constexpr int kDecodeWarps = 8;             // two threads per weight row
constexpr int kDecoders = kDecodeWarps * 32;
constexpr int kThreads = 32 + kDecoders + 32;  // producer warp, decode warps, MMA warp
constexpr int kMmaWarp = 1 + kDecodeWarps;
constexpr int kTmemCols = 128;
constexpr int kSpinLimit = 1 << 24;
// shared memory: kUStages weight units (nibbles with 128-byte swizzle, then scale codes), kABuf
// decoded tiles, then as many x tiles (N rows of 128 bytes, 128-byte swizzle) as the CTA's
// share holds, at most kStages; N is a multiple of 16, so every piece keeps the 1024-byte
// alignment of the swizzle
__host__ __device__ constexpr size_t fixed_bytes() {
    return 1024 + (size_t)kUStages * kUnitBytes + (size_t)kABuf * kABytes;
}
__host__ __device__ constexpr int x_stages(int nx) {
    return (int)((kCtaSmemBudget - fixed_bytes()) / ((size_t)nx * kXRowBytes)) > kStages
               ? kStages
               : (int)((kCtaSmemBudget - fixed_bytes()) / ((size_t)nx * kXRowBytes));
}
constexpr size_t smem_bytes(int nx) {
    return fixed_bytes() + (size_t)x_stages(nx) * nx * kXRowBytes;
}
constexpr size_t kSmemMax = kCtaSmemBudget;
static_assert(x_stages(kMaxXRows) >= 2, "the x ring needs two tiles at N = 128");

struct TcParams {
    uint16_t* y;        // bf16 [M][ldy] when splits == 1; null: fp32 partial tiles instead
    int64_t ldy;
    int64_t n, k;
    int m;
    int nx;             // MMA N: M rounded up to 16
    uint32_t idesc;     // instruction descriptor for that N
    float g;
    const float* descale;  // [M]: 2^-e(m) of the f16 copy of x
    int tiles;
    int splits;
    int units;          // 256-k units along K
    float* partial;     // [tiles][splits][M][128] fp32 (splits > 1)
    int32_t* error;
};

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

// Bounded wait for the phase with the given parity; false after the limit.
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

// Shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row atoms 1024 bytes apart.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)1 << 16) |
           ((uint64_t)(1024 >> 4) << 32) | ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// Instruction descriptor of kind::f16: D fp32, A and B f16, both K-major, M = 128, N = nx.
inline uint32_t idesc_f16(int nx) {
    return (1u << 4) | ((uint32_t)(nx >> 3) << 17) | ((uint32_t)(kRows >> 4) << 24);
}

__device__ __forceinline__ void mma_f16(uint32_t tmem, uint64_t adesc, uint64_t bdesc,
                                        uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate));
}

__device__ __forceinline__ void mma_commit(uint64_t* bar) {
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
            smem_u32(bar))
        : "memory");
}

// Two e4m3 codes (low byte first) -> f16x2, exact.
__device__ __forceinline__ uint32_t scale_pair(uint32_t codes) {
    uint32_t h;
    asm("{\n\t.reg .b16 t;\n\tcvt.u16.u32 t, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, t;\n\t}"
        : "=r"(h)
        : "r"(codes));
    return h;
}

// 8 e2m1 nibbles of a word (nibble i = k i, low nibble first) times an f16 scale (both halves
// equal) -> 4 f16x2 words {k 2i, k 2i+1}, exact (at most 6 significant bits).
__device__ __forceinline__ uint4 decode_word_f16(uint32_t w, uint32_t scl) {
    uint32_t h[4];
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\tmov.b32 {b0, b1, b2, b3}, %4;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, b0;\n\tcvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %2, b2;\n\tcvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
        : "=r"(h[0]), "=r"(h[1]), "=r"(h[2]), "=r"(h[3])
        : "r"(w));
#pragma unroll
    for (int i = 0; i < 4; ++i) asm("mul.rn.f16x2 %0, %0, %1;" : "+r"(h[i]) : "r"(scl));
    return make_uint4(h[0], h[1], h[2], h[3]);
}

__device__ __forceinline__ uint16_t f2bf(float v) {
    uint32_t u;
    asm("{\n\t.reg .b16 h;\n\tcvt.rn.bf16.f32 h, %1;\n\tmov.b32 %0, {h, h};\n\t}"
        : "=r"(u)
        : "f"(v));
    return (uint16_t)u;
}

__global__ void __launch_bounds__(kThreads, kCtasPerSm)
    nvfp4_tc_kernel(const TcParams p, const __grid_constant__ CUtensorMap tx,
                    const __grid_constant__ CUtensorMap tw, const __grid_constant__ CUtensorMap ts) {
    extern __shared__ __align__(16) uint8_t smem_raw[];
    uint8_t* const base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const int xbytes = p.nx * kXRowBytes;               // x tile of a stage
    uint8_t* const uring = base;                        // kUStages weight units
    uint8_t* const abuf = base + kUStages * kUnitBytes; // kABuf decoded tiles
    uint8_t* const xring = abuf + kABuf * kABytes;      // kStages x tiles
    __shared__ __align__(8) uint64_t xfull_bar[kStages], xempty_bar[kStages],
        ufull_bar[kUStages], uempty_bar[kUStages], afull_bar[kABuf], aempty_bar[kABuf], done_bar;
    __shared__ uint32_t tmem_base;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int xst = x_stages(p.nx);  // x ring depth
    const int tile = blockIdx.x / p.splits, split = blockIdx.x - tile * p.splits;
    const int u_begin = (int)((int64_t)p.units * split / p.splits);
    const int u_end = (int)((int64_t)p.units * (split + 1) / p.splits);
    const int stages = (u_end - u_begin) * kSub;

    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(&tmem_base)),
                     "r"(kTmemCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    if (tid == 0) {
        for (int i = 0; i < kStages; ++i) {
            mbar_init(&xfull_bar[i], 1);
            mbar_init(&xempty_bar[i], 1);  // the MMA commit
        }
        for (int i = 0; i < kUStages; ++i) {
            mbar_init(&ufull_bar[i], 1);
            mbar_init(&uempty_bar[i], kDecoders);  // every decoder, after the unit's last stage
        }
        for (int i = 0; i < kABuf; ++i) {
            mbar_init(&afull_bar[i], kDecoders);
            mbar_init(&aempty_bar[i], 1);
        }
        mbar_init(&done_bar, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    const uint32_t tmem = tmem_base;
    bool ok = true;

    if (warp == 0) {
        // ---- producer: a weight unit (nibbles and scale codes) every kSub stages, an x tile
        // every stage
        if (lane == 0) {
            for (int s = 0; s < stages && ok; ++s) {
                if (s % kSub == 0) {
                    const int u = s / kSub, us = u % kUStages;
                    if (u >= kUStages && !mbar_wait(&uempty_bar[us], ((u / kUStages) - 1) & 1)) {
                        ok = false;
                        break;
                    }
                    uint8_t* dst = uring + us * kUnitBytes;
                    mbar_expect_tx(&ufull_bar[us], (uint32_t)kUnitBytes);
                    tma_load_2d(dst, &tw, (u_begin + u) * (kUnitK / 2), tile * kRows, &ufull_bar[us]);
                    tma_load_2d(dst + kWBytes, &ts, (u_begin + u) * 16, tile * kRows, &ufull_bar[us]);
                }
                const int slot = s % xst;
                if (s >= xst && !mbar_wait(&xempty_bar[slot], ((s / xst) - 1) & 1)) {
                    ok = false;
                    break;
                }
                mbar_expect_tx(&xfull_bar[slot], (uint32_t)xbytes);
                tma_load_2d(xring + slot * xbytes, &tx, u_begin * kUnitK + s * kStageK, 0,
                            &xfull_bar[slot]);
            }
            if (!ok) atomicExch(p.error, 4);
        }
    } else if (warp == kMmaWarp) {
        // ---- MMA issuer
        if (lane == 0) {
            for (int s = 0; s < stages && ok; ++s) {
                const int slot = s % xst, buf = s % kABuf;
                if (!mbar_wait(&xfull_bar[slot], (s / xst) & 1) ||
                    !mbar_wait(&afull_bar[buf], (s / kABuf) & 1)) {
                    ok = false;
                    break;
                }
                asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
                const uint32_t a0 = smem_u32(abuf + buf * kABytes);
                const uint32_t b0 = smem_u32(xring + slot * xbytes);
#pragma unroll
                for (int kk = 0; kk < kStageK / 16; ++kk)
                    mma_f16(tmem, sw128_desc(a0 + kk * 32), sw128_desc(b0 + kk * 32), p.idesc,
                            (s > 0 || kk > 0) ? 1u : 0u);
                mma_commit(&aempty_bar[buf]);
                mma_commit(&xempty_bar[slot]);
            }
            if (ok) mma_commit(&done_bar);
            else atomicExch(p.error, 5);
        }
    } else {
        // ---- decoders: threads 2r and 2r+1 decode the two 32-k halves of weight row r of
        // every 64-k stage
        const int d = tid - 32, r = d >> 1, half = d & 1;
        for (int s = 0; s < stages && ok; ++s) {
            const int u = s / kSub, sub = s % kSub, us = u % kUStages, buf = s % kABuf;
            if (!mbar_wait(&ufull_bar[us], (u / kUStages) & 1) ||
                (s >= kABuf && !mbar_wait(&aempty_bar[buf], ((s / kABuf) - 1) & 1))) {
                ok = false;
                break;
            }
            const uint8_t* unit = uring + us * kUnitBytes;
            // 16-byte chunk c = 2 sub + half of the row (k = 32 c .. 32 c + 31 of the unit),
            // 128-byte swizzle
            const int c = 2 * sub + half;
            const uint4 wv = *reinterpret_cast<const uint4*>(unit + r * 128 + ((c ^ (r & 7)) << 4));
            // this half's 2 scale codes of the stage's 4
            const uint32_t sc =
                *reinterpret_cast<const uint16_t*>(unit + kWBytes + r * 16 + sub * 4 + half * 2);
            if (sub == kSub - 1) mbar_arrive(&uempty_bar[us]);  // done with this unit
            const uint32_t s01 = scale_pair(sc);
            const uint32_t s0 = __byte_perm(s01, 0, 0x1010), s1 = __byte_perm(s01, 0, 0x3232);
            uint8_t* row = abuf + buf * kABytes + (r >> 3) * 1024 + (r & 7) * 128;
            // words j hold stage k = 32 half + 8 j .. +8: decoded chunk 4 half + j of the A row
            const uint32_t words[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int cc = 4 * half + j;
                *reinterpret_cast<uint4*>(row + ((cc ^ (r & 7)) << 4)) =
                    decode_word_f16(words[j], j < 2 ? s0 : s1);
            }
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            mbar_arrive(&afull_bar[buf]);
        }
        if (!ok) atomicExch(p.error, 6);

        // ---- epilogue (decode warps 1..4): TMEM lane 32 (warp % 4) + lane is weight row rr;
        // column m is x row m
        if (warp <= 4) {
            bool done = ok && mbar_wait(&done_bar, 0);
            if (ok && !done) atomicExch(p.error, 7);
            done = __all_sync(0xFFFFFFFFu, done);  // tcgen05.ld is warp-wide
            asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
            const int rr = 32 * (warp & 3) + lane;
            const int64_t n = (int64_t)tile * kRows + rr;
            if (done) {
                for (int c0 = 0; c0 < p.m; c0 += 32) {
                    uint32_t v[32];
                    const uint32_t taddr =
                        tmem + ((uint32_t)(32 * (warp & 3)) << 16) + (uint32_t)c0;
                    asm volatile(
                        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
                        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
                        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
                        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]),
                          "=r"(v[6]), "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]),
                          "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]),
                          "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]),
                          "=r"(v[21]), "=r"(v[22]), "=r"(v[23]), "=r"(v[24]), "=r"(v[25]),
                          "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]),
                          "=r"(v[31])
                        : "r"(taddr));
                    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
                    if (n < p.n) {
                        const int cols = p.m - c0 < 32 ? p.m - c0 : 32;
                        if (p.splits == 1 && p.y) {
#pragma unroll
                            for (int j = 0; j < 32; ++j)
                                if (j < cols)
                                    p.y[(int64_t)(c0 + j) * p.ldy + n] = f2bf(
                                        __uint_as_float(v[j]) * p.descale[c0 + j] * p.g);
                        } else {
                            float* part =
                                p.partial + ((int64_t)blockIdx.x * p.m + c0) * kRows + rr;
#pragma unroll
                            for (int j = 0; j < 32; ++j)
                                if (j < cols) part[(int64_t)j * kRows] = __uint_as_float(v[j]);
                        }
                    }
                }
            }
        }
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    if (warp == 0)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                     "r"(kTmemCols));
}

// The partial tiles of a K split, added in split order: element (m, n) of tile t, split j is
// partial[((t splits + j) M + m) 128 + n % 128].  Grid: blockIdx.y = row m of x, 4 consecutive
// outputs per thread (float4 loads; a tile is 128 outputs, so the 4 share a tile).

constexpr int kReduceThreads = 256;

// y[m][n] = bf16(g * 2^-e(m) * sum of the partials)
__global__ void __launch_bounds__(kReduceThreads)
    nvfp4_tc_reduce(const float* __restrict__ partial, const float* __restrict__ descale,
                    uint16_t* y, int64_t ldy, int64_t n, int m, float g, int splits) {
    const int mm = blockIdx.y;
    const int64_t n0 = ((int64_t)blockIdx.x * kReduceThreads + threadIdx.x) * 4;
    if (n0 >= n) return;
    const int64_t tile = n0 / kRows;
    const int r = (int)(n0 - tile * kRows);
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    for (int j = 0; j < splits; ++j) {
        const float4 v = *reinterpret_cast<const float4*>(
            partial + (((tile * splits + j) * (int64_t)m) + mm) * kRows + r);
        acc[0] += v.x;
        acc[1] += v.y;
        acc[2] += v.z;
        acc[3] += v.w;
    }
    const float ds = descale[mm];
#pragma unroll
    for (int i = 0; i < 4; ++i)
        if (n0 + i < n) y[(int64_t)mm * ldy + n0 + i] = f2bf(acc[i] * ds * g);
}

// The dual's last pass over both streams' partials:
//   o[m][n] = bf16(silu(g_g 2^-e(m) gate) * (g_u 2^-e(m) up)),  silu(t) = t / (1 + e^-t), fp32
__global__ void __launch_bounds__(kReduceThreads)
    nvfp4_tc_dual_finish(const float* __restrict__ pg, const float* __restrict__ pu,
                         const float* __restrict__ descale, uint16_t* y, int64_t ldy, int64_t n,
                         int m, float gg, float gu, int splits) {
    const int mm = blockIdx.y;
    const int64_t n0 = ((int64_t)blockIdx.x * kReduceThreads + threadIdx.x) * 4;
    if (n0 >= n) return;
    const int64_t tile = n0 / kRows;
    const int r = (int)(n0 - tile * kRows);
    float ag[4] = {0.f, 0.f, 0.f, 0.f}, au[4] = {0.f, 0.f, 0.f, 0.f};
    for (int j = 0; j < splits; ++j) {
        const int64_t off = (((tile * splits + j) * (int64_t)m) + mm) * kRows + r;
        const float4 a = *reinterpret_cast<const float4*>(pg + off);
        const float4 b = *reinterpret_cast<const float4*>(pu + off);
        ag[0] += a.x;
        ag[1] += a.y;
        ag[2] += a.z;
        ag[3] += a.w;
        au[0] += b.x;
        au[1] += b.y;
        au[2] += b.z;
        au[3] += b.w;
    }
    const float ds = descale[mm];
#pragma unroll
    for (int i = 0; i < 4; ++i)
        if (n0 + i < n) {
            const float a = ag[i] * ds * gg, b = au[i] * ds * gu;
            y[(int64_t)mm * ldy + n0 + i] = f2bf(a / (1.0f + expf(-a)) * b);
        }
}

// The f16 copy of x (after the call's prologue, if any): row m scaled by 2^e(m) so that its
// largest magnitude lands in [2^14, 2^15) (exact for every bf16 value at most 2^24 times
// smaller), and 2^-e(m).  One block per row, 16-byte accesses (K % 256 == 0, 16-byte aligned
// rows).  With the residual-add + RMS-norm prologue the block first sums h^2 over the row (a
// fixed xor tree per warp, then the warps in order) and writes h.
__global__ void __launch_bounds__(512) nvfp4_tc_prep(const uint16_t* __restrict__ x, int64_t ldx,
                                                     int64_t k, uint16_t* x16, float* descale,
                                                     const nvfp4_pro::Prologue pro) {
    const int m = blockIdx.x;
    const uint4* row = reinterpret_cast<const uint4*>(x + (int64_t)m * ldx);
    const int64_t k8 = k / 8;
    __shared__ uint32_t red[32];
    __shared__ float fred[32];
    float inv = 0.f;
    if (pro.kind == NVFP4_PROLOGUE_ADD_RMSNORM) {
        const uint4* rr = reinterpret_cast<const uint4*>(pro.in + (int64_t)m * pro.ld_in);
        uint4* hr = pro.hout ? reinterpret_cast<uint4*>(pro.hout + (int64_t)m * pro.ldh) : nullptr;
        float ss = 0.f;
        for (int64_t i = threadIdx.x; i < k8; i += blockDim.x) {
            const uint4 h = nvfp4_pro::add_8(row[i], rr[i]);
            ss = nvfp4_pro::sum_squares_8(h, ss);
            if (hr) hr[i] = h;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xFFFFFFFFu, ss, o);
        if ((threadIdx.x & 31) == 0) fred[threadIdx.x >> 5] = ss;
        __syncthreads();
        if (threadIdx.x == 0) {
            float t = 0.f;
            for (int w = 0; w < (int)(blockDim.x >> 5); ++w) t += fred[w];
            fred[0] = nvfp4_pro::rms_inverse(t, k, pro.eps);
        }
        __syncthreads();
        inv = fred[0];
    }
    uint32_t a = 0;
    for (int64_t i = threadIdx.x; i < k8; i += blockDim.x) {
        uint4 v = row[i];
        if (pro.kind != NVFP4_PROLOGUE_NONE) v = nvfp4_pro::apply_8(pro, v, m, 8 * i, inv);
        // per-halfword maximum (two bf16 magnitudes per word), folded below
        a = __vmaxu2(a, __vmaxu2(__vmaxu2(v.x & 0x7FFF7FFFu, v.y & 0x7FFF7FFFu),
                                 __vmaxu2(v.z & 0x7FFF7FFFu, v.w & 0x7FFF7FFFu)));
    }
    a = max(a & 0xFFFFu, a >> 16);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) a = max(a, __shfl_xor_sync(0xFFFFFFFFu, a, o));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = a;
    __syncthreads();
    if (threadIdx.x < 32) {
        a = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0u;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) a = max(a, __shfl_xor_sync(0xFFFFFFFFu, a, o));
        if (threadIdx.x == 0) red[0] = a;
    }
    __syncthreads();
    a = red[0];
    int e = 0;
    if (a != 0u && a < 0x7F80u) e = 14 - ((int)(a >> 7) - 127);
    e = e > 126 ? 126 : (e < -126 ? -126 : e);
    const float sc = __uint_as_float((uint32_t)(e + 127) << 23);
    if (threadIdx.x == 0) descale[m] = __uint_as_float((uint32_t)(127 - e) << 23);
    uint4* out = reinterpret_cast<uint4*>(x16 + (int64_t)m * k);
    for (int64_t i = threadIdx.x; i < k8; i += blockDim.x) {
        uint4 v = row[i];
        if (pro.kind != NVFP4_PROLOGUE_NONE) v = nvfp4_pro::apply_8(pro, v, m, 8 * i, inv);
        const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
        uint32_t h4[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const __half2 t = __floats2half2_rn(__uint_as_float(w4[j] << 16) * sc,
                                                __uint_as_float(w4[j] & 0xFFFF0000u) * sc);
            h4[j] = *reinterpret_cast<const uint32_t*>(&t);
        }
        out[i] = make_uint4(h4[0], h4[1], h4[2], h4[3]);
    }
}

}  // namespace

// ------------------------------------------------------------------------------------------
// host side (called from the C ABI in nvfp4_gemv.cu)

namespace nvfp4_tc {

#ifndef NVFP4_TC_ITEM_COST
#define NVFP4_TC_ITEM_COST 2
#endif
// splits: the fewest that minimise the makespan: the waves a CTA runs (ceil(items / (2 sms)),
// two CTAs per SM) times the cost of an item, its units plus a fixed cost of NVFP4_TC_ITEM_COST
// units (start-up, the pipeline's fill and drain, writing the partials).  Depends only on (N, K,
// SM count).
int choose_splits(int64_t n, int64_t k, int sms) {
    const int64_t tiles = (n + kRows - 1) / kRows;
    const int64_t units = (k + kUnitK - 1) / kUnitK;
    int best = 1;
    int64_t best_cost = -1;
    for (int s = 1; s <= 32 && s <= units; ++s) {
        const int64_t waves = (tiles * s + kCtasPerSm * sms - 1) / (kCtasPerSm * sms);
        const int64_t per = (units + s - 1) / s;
        const int64_t cost = waves * (per + NVFP4_TC_ITEM_COST);
        if (best_cost < 0 || cost < best_cost) {
            best_cost = cost;
            best = s;
        }
    }
    return best;
}

static size_t align256(size_t v) { return (v + 255) / 256 * 256; }

// fp32 partial tiles of one weight's call: when its K is split, and always for the dual's
// streams (their last pass reads both)
static size_t partial_bytes(int64_t n, int64_t k, int m, int sms, bool always = false) {
    const int64_t tiles = (n + kRows - 1) / kRows;
    const int splits = choose_splits(n, k, sms);
    return (splits > 1 || always) ? (size_t)tiles * splits * m * kRows * sizeof(float) : 0;
}

// Scratch of a call: fp32 partial tiles (the dual: one set per stream), the f16 copy of x and
// the row descales.
struct Scratch {
    size_t partial, partial_up, x16, descale, total;
};

static Scratch scratch_layout(int64_t n, int64_t k, int m, int sms, bool dual) {
    Scratch sc;
    const size_t pb = align256(partial_bytes(n, k, m, sms, dual));
    sc.partial = 0;
    sc.partial_up = pb;
    sc.x16 = dual ? 2 * pb : pb;
    sc.descale = sc.x16 + align256((size_t)m * k * 2);
    sc.total = sc.descale + align256((size_t)m * sizeof(float));
    return sc;
}

size_t scratch_bytes(int64_t n, int64_t k, int m, int sms) {
    return scratch_layout(n, k, m, sms, true).total;  // covers the single and the dual
}

bool usable(const void* s, int64_t k) {
    return (k % kUnitK) == 0 && (reinterpret_cast<uintptr_t>(s) & 15u) == 0;
}

static int set_attr() {
    static bool attr_set[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
        cudaGetLastError();
        return NVFP4_ERR_ARCH;
    }
    if (!attr_set[dev]) {
        // the whole shared-memory carveout, so that two CTAs' shares fit on an SM
        if (cudaFuncSetAttribute(nvfp4_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)kSmemMax) != cudaSuccess ||
            cudaFuncSetAttribute(nvfp4_tc_kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                                 100) != cudaSuccess) {
            cudaGetLastError();
            return NVFP4_ERR_LAUNCH;
        }
        attr_set[dev] = true;
    }
    return NVFP4_OK;
}

// The weight's tile pass over the f16 copy of x (already written), then the split reduction.
static int enqueue_weight(EncodeFn encode, int sms, const uint8_t* w, const uint8_t* s, float g,
                          const uint16_t* x16, const float* descale, float* partial, int m, int64_t n,
                          int64_t k, uint16_t* y, int64_t ldy, int32_t* error,
                          cudaStream_t stream) {
    const int tiles = (int)((n + kRows - 1) / kRows);
    const int splits = choose_splits(n, k, sms);
    const int nx = (m + 15) / 16 * 16;  // MMA N
    CUtensorMap tx, tw, ts;
    memset(&tx, 0, sizeof(tx));
    memset(&tw, 0, sizeof(tw));
    memset(&ts, 0, sizeof(ts));
    const cuuint32_t one[2] = {1, 1};
    {
        // the f16 copy of x: [M][K], box 64 k x N rows, 128-byte swizzle; rows >= M read as zero
        const cuuint64_t dims[2] = {(cuuint64_t)k, (cuuint64_t)m};
        const cuuint64_t strides[1] = {(cuuint64_t)k * 2};
        const cuuint32_t box[2] = {(cuuint32_t)kStageK, (cuuint32_t)nx};
        if (encode(&tx, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<uint16_t*>(x16), dims,
                   strides, box, one, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) !=
            CUDA_SUCCESS)
            return NVFP4_ERR_LAUNCH;
    }
    {
        const cuuint64_t dims[2] = {(cuuint64_t)(k / 2), (cuuint64_t)n};
        const cuuint64_t strides[1] = {(cuuint64_t)(k / 2)};
        const cuuint32_t box[2] = {(cuuint32_t)(kUnitK / 2), (cuuint32_t)kRows};
        if (encode(&tw, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(w), dims, strides,
                   box, one, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) !=
            CUDA_SUCCESS)
            return NVFP4_ERR_LAUNCH;
    }
    {
        const cuuint64_t dims[2] = {(cuuint64_t)(k / 16), (cuuint64_t)n};
        const cuuint64_t strides[1] = {(cuuint64_t)(k / 16)};
        const cuuint32_t box[2] = {16, (cuuint32_t)kRows};
        if (encode(&ts, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(s), dims, strides,
                   box, one, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) !=
            CUDA_SUCCESS)
            return NVFP4_ERR_LAUNCH;
    }
    TcParams p;
    memset(&p, 0, sizeof(p));
    p.y = y;
    p.ldy = ldy;
    p.n = n;
    p.k = k;
    p.m = m;
    p.nx = nx;
    p.idesc = idesc_f16(nx);
    p.g = g;
    p.descale = descale;
    p.tiles = tiles;
    p.splits = splits;
    p.units = (int)((k + kUnitK - 1) / kUnitK);
    p.error = error;
    p.partial = partial;
    nvfp4_tc_kernel<<<tiles * splits, kThreads, smem_bytes(nx), stream>>>(p, tx, tw, ts);
    if (cudaGetLastError() != cudaSuccess) return NVFP4_ERR_LAUNCH;
    if (splits > 1 && y) {
        const dim3 grid((unsigned)((n + 4 * kReduceThreads - 1) / (4 * kReduceThreads)),
                        (unsigned)m);
        nvfp4_tc_reduce<<<grid, kReduceThreads, 0, stream>>>(partial, descale, y, ldy, n, m, g,
                                                             splits);
        if (cudaGetLastError() != cudaSuccess) return NVFP4_ERR_LAUNCH;
    }
    return NVFP4_OK;
}

int launch(EncodeFn encode, int sms, const uint8_t* w, const uint8_t* s, float g, const void* x,
           int64_t ldx, void* y, int64_t ldy, int m, int64_t n, int64_t k,
           const nvfp4_pro::Prologue& pro, void* ws, size_t ws_bytes, size_t scratch_off,
           cudaStream_t stream) {
    if (ws_bytes < scratch_off + scratch_bytes(n, k, m, sms)) return NVFP4_ERR_WORKSPACE;
    int st = set_attr();
    if (st != NVFP4_OK) return st;
    const Scratch sc = scratch_layout(n, k, m, sms, false);
    char* const base = static_cast<char*>(ws) + scratch_off;
    uint16_t* const x16 = reinterpret_cast<uint16_t*>(base + sc.x16);
    float* const descale = reinterpret_cast<float*>(base + sc.descale);
    nvfp4_tc_prep<<<m, 512, 0, stream>>>(static_cast<const uint16_t*>(x), ldx, k, x16, descale,
                                         pro);
    if (cudaGetLastError() != cudaSuccess) return NVFP4_ERR_LAUNCH;
    return enqueue_weight(encode, sms, w, s, g, x16, descale,
                          reinterpret_cast<float*>(base + sc.partial), m, n, k,
                          static_cast<uint16_t*>(y), ldy, static_cast<int32_t*>(ws), stream);
}

int launch_dual(EncodeFn encode, int sms, const uint8_t* wg, const uint8_t* sg, float gg,
                const uint8_t* wu, const uint8_t* su, float gu, const void* x, int64_t ldx,
                void* y, int64_t ldy, int m, int64_t n, int64_t k, const nvfp4_pro::Prologue& pro,
                void* ws, size_t ws_bytes, size_t scratch_off, cudaStream_t stream) {
    if (ws_bytes < scratch_off + scratch_bytes(n, k, m, sms)) return NVFP4_ERR_WORKSPACE;
    int st = set_attr();
    if (st != NVFP4_OK) return st;
    const Scratch sc = scratch_layout(n, k, m, sms, true);
    char* const base = static_cast<char*>(ws) + scratch_off;
    uint16_t* const x16 = reinterpret_cast<uint16_t*>(base + sc.x16);
    float* const descale = reinterpret_cast<float*>(base + sc.descale);
    float* const pg = reinterpret_cast<float*>(base + sc.partial);
    float* const pu = reinterpret_cast<float*>(base + sc.partial_up);
    int32_t* const error = static_cast<int32_t*>(ws);
    nvfp4_tc_prep<<<m, 512, 0, stream>>>(static_cast<const uint16_t*>(x), ldx, k, x16, descale,
                                         pro);
    if (cudaGetLastError() != cudaSuccess) return NVFP4_ERR_LAUNCH;
    // both streams as fp32 partial tiles (y null), then one pass forms o
    if ((st = enqueue_weight(encode, sms, wg, sg, gg, x16, descale, pg, m, n, k, nullptr, 0,
                             error, stream)) != NVFP4_OK)
        return st;
    if ((st = enqueue_weight(encode, sms, wu, su, gu, x16, descale, pu, m, n, k, nullptr, 0,
                             error, stream)) != NVFP4_OK)
        return st;
    const dim3 grid((unsigned)((n + 4 * kReduceThreads - 1) / (4 * kReduceThreads)), (unsigned)m);
    nvfp4_tc_dual_finish<<<grid, kReduceThreads, 0, stream>>>(
        pg, pu, descale, static_cast<uint16_t*>(y), ldy, n, m, gg, gu, choose_splits(n, k, sms));
    if (cudaGetLastError() != cudaSuccess) return NVFP4_ERR_LAUNCH;
    return NVFP4_OK;
}

int launch_multi(EncodeFn encode, int sms, const uint8_t* const* w, const uint8_t* const* s,
                 const float* g, void* const* y, const int64_t* ldy, const int64_t* n, int count,
                 const void* x, int64_t ldx, int m, int64_t k, const nvfp4_pro::Prologue& pro,
                 void* ws, size_t ws_bytes, size_t scratch_off, cudaStream_t stream) {
    // one f16 copy of x for every output, after the partial tiles of the largest split
    size_t need = 0, pmax = 0;
    for (int o = 0; o < count; ++o) {
        const size_t b = scratch_bytes(n[o], k, m, sms), pb = partial_bytes(n[o], k, m, sms);
        need = b > need ? b : need;
        pmax = pb > pmax ? pb : pmax;
    }
    if (ws_bytes < scratch_off + need) return NVFP4_ERR_WORKSPACE;
    int st = set_attr();
    if (st != NVFP4_OK) return st;
    char* const base = static_cast<char*>(ws) + scratch_off;
    float* const partial = reinterpret_cast<float*>(base);
    uint16_t* const x16 = reinterpret_cast<uint16_t*>(base + align256(pmax));
    float* const descale =
        reinterpret_cast<float*>(base + align256(pmax) + align256((size_t)m * k * 2));
    nvfp4_tc_prep<<<m, 512, 0, stream>>>(static_cast<const uint16_t*>(x), ldx, k, x16, descale,
                                         pro);
    if (cudaGetLastError() != cudaSuccess) return NVFP4_ERR_LAUNCH;
    for (int o = 0; o < count; ++o)
        if ((st = enqueue_weight(encode, sms, w[o], s[o], g[o], x16, descale, partial, m, n[o], k,
                                 static_cast<uint16_t*>(y[o]), ldy[o],
                                 static_cast<int32_t*>(ws), stream)) != NVFP4_OK)
            return st;
    return NVFP4_OK;
}

}  // namespace nvfp4_tc
