// Weight-only NVFP4 GEMV / fused dual GEMV / multi-output GEMV / chained GEMVs for NVIDIA B200
// (sm_100a), with its C ABI.
//
// The operation is the "w4a16_gemv" / "w4a16_gemv_dual" kernel family of a hybrid decoder's
// decode step ("Blueprint - circuit executor" page for qwen3.8-27b-nvfp4 on GB10, table
// "Kernels the plan launches"; weight format "nvfp4/g16", activations bf16, table "Weighted
// nodes"); the fused SiLU(gate)*up epilogue replaces that plan's separate "moe_silu_mul" launch
// (planner setting decode_split_silu).  The multi-output form runs up to four weights that share
// x in one launch (that plan's two-output k/v and q+gate GEMVs), and a chain runs up to 16 such
// operations back to back in one launch, an operation reading the result of an earlier one as
// its x (the MLP's gate_up dual feeding down).  Row counts 1..8 per pass (8-row speculative
// draft/verify round, kern-qwen38-sm103 model card, section "Run"); calls of up to 128 rows
// (the plan's multi_seq arms) run one pass per 8 rows.  Formats and the ABI are in nvfp4.h.
//
// Design (B200-first):
//   * The path is HBM-bound: 0.5625 bytes per weight.  A persistent grid (one CTA per SM)
//     splits each operation's work -- units of 128 output rows x 256 k in row-group-major
//     order -- into equal contiguous ranges ("stream-K"), so every SM streams the same number
//     of bytes.  The split depends only on (N, K, SM count), never on M.
//   * A row group cut by range boundaries is finished by the CTA holding its first unit (the
//     owner), which reaches it at the end of its range: the later CTAs of the group publish their
//     fp32 partial sums early in their ranges and count themselves in on the group's hand-off
//     word, and the owner adds them in CTA order.  The owner waits for them at most 50 us: if
//     they are not all there (not resident because other work holds SMs) it publishes its own
//     partial sums and marks the word, and the last of them to arrive finishes the group
//     instead.  One read-modify-write word per group orders all of it, so exactly one CTA
//     finishes each group, nothing waits without bound, and the sum's order (hence every bit of
//     the result) is fixed by the split.
//   * A producer warp streams each unit with TMA (cp.async.bulk.tensor, no multicast, L2
//     evict-first): one 128-row x 128-byte box of packed weights (128-byte swizzle) and one
//     128-row x 16-byte box of scale codes per weight stream.  A ring entry of shared memory,
//     guarded by one pair of mbarriers, holds two of these 18 KB halves: the dual's gate and up
//     of one unit, or two consecutive units of a single-stream operation.  When the scale rows
//     cannot be moved by TMA (K % 256 != 0 or misaligned) the producer lanes copy them with
//     cp.async.  Boxes past N or K are zero-filled.  In a chain the producer runs ahead across
//     operation boundaries: the weights do not depend on earlier results.
//   * Decode in registers with the hardware conversions: cvt e2m1x2 -> f16x2 turns each byte
//     (two nibbles, k and k+1) into an f16 pair, cvt e4m3x2 -> f16x2 turns two scale codes into
//     f16, and one f16x2 multiply gives A = e2m1 * e4m3, exact in f16 (at most 6 significant
//     bits, magnitude in [2^-10, 2688] or zero).
//   * The dot products run on the tensor cores: mma.m16n8k16 (f16 in, fp32 accumulate) with
//     16 weight rows as A and x as B, padded to 8 columns (columns >= M are zero).  The same
//     instruction sequence serves every M, so row m of the output depends only on x row m:
//     bitwise row invariance across M = 1..8, and across 1..128 with the 8-row passes.  Within a
//     16-row tile the mma's row r is weight row perm(r) (rows r and r+1 four apart), which
//     makes the swizzled reads conflict-free.
//   * x is staged per operation and CTA in shared memory as f16 (cp.async, then converted in
//     place, each row by its own warps).  Each x row m is scaled by a power of two 2^e(m) chosen
//     from the row's largest magnitude in the CTA's k range (so it lands in [2^14, 2^15)); bf16
//     values convert exactly unless they are more than 2^31 times smaller than that maximum.
//     The partial sums are multiplied back by 2^-e(m) (exact) before they are combined.  The
//     producer issues at most kPrefetch units of weights before the consumers have requested
//     their first x: a longer queue of weight boxes ahead of those requests would delay them.
//   * Chains: an operation that reads an earlier one's result waits (bounded, acquire) until
//     that operation's completed-row-group count is full; every CTA adds the groups it finished
//     (release) at the end of its range.  Such chains are launched cooperatively, so all CTAs
//     are resident together and those waits end.
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

constexpr int kBlockK = 128;                      // k per mma block (4 lanes x 32) and per x slot
constexpr int kUnitK = 256;                       // k per unit
constexpr int kWRowBytes = kUnitK / 2;            // 128 bytes of packed W per row and unit
constexpr int kSRowBytes = kUnitK / 16;           // 16 scale codes per row and unit
constexpr int kConsumerWarps = 8;                 // each owns 16 rows of a unit
constexpr int kConsumers = kConsumerWarps * 32;
constexpr int kThreads = kConsumers + 32;         // + one producer warp
constexpr int kRows = kConsumerWarps * 16;        // 128 output rows per unit
constexpr int kWBytes = kRows * kWRowBytes;       // packed weights of one unit and stream
constexpr int kSBytes = kRows * kSRowBytes;       // scale codes of one unit and stream
constexpr int kSlotBytes = kWBytes + kSBytes;     // one unit of one weight stream: 18 KB
// A ring entry holds two of them under one pair of barriers: the dual's gate and up of one unit,
// or two consecutive units of a single-stream operation (the last entry of a range may hold one).
constexpr int kEntryBytes = 2 * kSlotBytes;
constexpr int kSlotU4 = 16;                       // uint4 of x per 128-k block per row
constexpr int kRowPadU4 = 4;                      // 64-byte pad between x rows (bank offset)
constexpr int kSmemMax = 225 * 1024;             // dynamic; + static shared memory <= 227 KB
constexpr int kPartialFloats = kRows * 8;         // one stream's partial tile (4 KB)
constexpr int kSpinLimit = 1 << 24;               // bounded mbarrier waits
constexpr int64_t kMaxK = int64_t(1) << 24;
constexpr int kMaxSlots = 6;                      // ring entries
// The row split of a launch is sized so that x fits beside a ring of kMinStages units; a
// launch uses as many slots as its shared memory allows (up to kMaxSlots), which does not
// change the arithmetic.
constexpr int kMinStages = 4;
// Units of weights issued before the consumers have requested their first x (which may wait
// for the preceding kernel): a longer queue of weight boxes ahead of those requests delays them.
constexpr int kPrefetch = 2;
constexpr int kMaxOutputs = NVFP4_MAX_OUTPUTS;
constexpr int kMaxChainOps = NVFP4_CHAIN_MAX_OPS;
constexpr int kChainMaps = 64;                    // tensor maps of one chain launch
constexpr int64_t kDefaultWaitNs = 1000000000;    // a chain's dependency waits give up after 1 s
// The hand-off word of a row group cut by range boundaries (indexed by the CTA holding its first
// unit, the owner): the number of later CTAs that have published their partial tiles, and
// kOwnerGone once the owner stopped waiting for them.  The owner waits for them at most
// kOwnerWaitNs: they are normally resident and done within a few microseconds; when they are
// not (other work holds SMs), waiting longer would only hold the owner's SM.
constexpr uint32_t kOwnerGone = 1u << 31;
constexpr int64_t kOwnerWaitNs = 50000;
static_assert(kSlotBytes % 1024 == 0, "slots must keep 1024-byte alignment (swizzle)");
static_assert(kEntryBytes % 1024 == 0, "entries must keep 1024-byte alignment (swizzle)");

enum ScaleMode { kScaleTma = 0, kScaleAsync8 = 1, kScaleScalar = 2 };
enum Mode { kModeSingle = 0, kModeDual = 1, kModeMulti = 2, kModeChain = 3 };

// Workspace: [0, 256) error word (int32 at 0) and a chain's exit count (uint32 at 4);
// [256, 512) a chain's completion counts, one uint32 per operation; then, per kernel operation,
// one hand-off word per CTA (padded to 256 bytes) and fp32 partial tiles [CTA][2][streams]
// (slot 0: a later CTA's head of a group, slot 1: the owner's tail when it stops waiting).
constexpr size_t kHeaderBytes = 512;
constexpr size_t kDoneOffset = 256;

// One operation of a launch.  Outputs of a single-stream operation are several weight matrices
// with the same K sharing x, their row groups concatenated in output order (one output for
// nvfp4_gemv); the dual has one output fed by two weight streams (index = stream).
struct Op {
    const uint16_t* x;
    int64_t ldx;
    int64_t k;
    int64_t units;                  // row groups * ku
    int ku;                         // 256-k units along K (the last may be partial)
    int grid;                       // CTAs the units are split over (<= the launch's grid)
    uint32_t uq, ur;                // units / grid and units % grid: CTA c's range starts at
                                    // floor(units c / grid) = uq c + (ur c) / grid
    int outs;                       // outputs (1 for the dual)
    int dual;
    int map0;                       // w / s tensor maps of output (stream) i: map0 + 2i, + 1
    int scale_mode;
    int wait_idx;                   // completion count to wait for before reading x, or -1
    uint32_t wait_target;           // row groups that count must reach
    int sig_idx;                    // completion count this operation adds to, or -1
    int rot;                        // the launch's CTA c works on range (c + rot) mod grid: a
                                    // chain turns the ranges by operation, so that no SM keeps
                                    // the same hand-off role in every layer
    const uint8_t* s[kMaxOutputs];  // scale codes, per output (dual: per stream)
    float g[kMaxOutputs];           // global scales, per output (dual: per stream)
    uint16_t* y[kMaxOutputs];       // outputs (dual: y[0])
    int64_t ldy[kMaxOutputs];
    int64_t n[kMaxOutputs];         // rows of each output (dual: n[0])
    int64_t gend[kMaxOutputs];      // row groups of outputs 0..o together
    uint32_t* arrive;               // [grid] hand-off words, by the CTA holding a group's first unit
    float* partial;                 // [grid][2][streams][kPartialFloats]
};

template <int OPS, int MAPS>
struct Launch {
    CUtensorMap maps[MAPS];         // packed weights and scale codes of every operation
    Op op[OPS];
    int ops;
    int m;
    int slots;                      // ring depth
    int full_count;                 // arrivals that complete a full slot: 1, or 33 when the
                                    // producer lanes copy the scale codes themselves
    int signals;                    // some operation signals completion (chains)
    int64_t wait_ns;                // limit of a dependency wait
    int64_t owner_wait_ns;          // limit of an owner's wait for the later CTAs' tiles
    uint32_t* done;                 // [kMaxChainOps] completion counts
    uint32_t* exit_count;
    int32_t* error;
};

template <int MODE>
struct ModeCfg {
    static constexpr int kOps = MODE == kModeChain ? kMaxChainOps : 1;
    static constexpr int kMaps = MODE == kModeChain ? kChainMaps
                                 : MODE == kModeSingle ? 2
                                 : MODE == kModeDual   ? 4
                                                       : 2 * kMaxOutputs;
};
template <int MODE>
using LaunchOf = Launch<ModeCfg<MODE>::kOps, ModeCfg<MODE>::kMaps>;

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

// L2 policy for the weight stream: read once, so it should not push x, y and the partial sums
// out of L2.
__device__ __forceinline__ uint64_t evict_first_policy() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y,
                                            uint64_t* bar, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
        ".L2::cache_hint [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar)), "l"(policy)
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

// Arrival on a count: the release half publishes this CTA's partial sums (ordered before it
// by a barrier), the acquire half makes the earlier arrivals' partial sums visible.
__device__ __forceinline__ uint32_t atom_add_acq_rel(uint32_t* p, uint32_t v) {
    uint32_t old;
    asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v)
                 : "memory");
    return old;
}

__device__ __forceinline__ uint32_t atom_or_acq_rel(uint32_t* p, uint32_t v) {
    uint32_t old;
    asm volatile("atom.acq_rel.gpu.global.or.b32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v)
                 : "memory");
    return old;
}

__device__ __forceinline__ void red_release_add(uint32_t* p, uint32_t v) {
    asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Bounded wait until *p >= target (acquire); false once limit_ns have passed.
__device__ __forceinline__ bool wait_count(const uint32_t* p, uint32_t target, int64_t limit_ns) {
    const uint64_t t0 = global_ns();
    for (int it = 0; it < kSpinLimit; ++it) {
        if (ld_acquire(p) >= target) return true;
        if ((int64_t)(global_ns() - t0) > limit_ns) return false;
        __nanosleep(64);
    }
    return false;
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

// A lane's decoded view of one unit half for one stream: the multiply-ready k-step operands.
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

// Output holding global row group rg (the groups of outputs 0..o end at op.gend[o]).
__device__ __forceinline__ int output_of(const Op& op, int64_t rg) {
    int o = 0;
    while (o + 1 < op.outs && rg >= op.gend[o]) ++o;
    return o;
}

// The CTA whose range of an operation's units holds unit u (ranges [U c / G, U (c+1) / G)).
__device__ __forceinline__ int cta_of(int64_t units, int grid, int64_t u) {
    return (int)(((u + 1) * grid + units - 1) / units) - 1;
}

// First unit of CTA c's range, floor(units c / grid), in 32-bit arithmetic (ur c < grid^2).
__device__ __forceinline__ int64_t range_begin(const Op& op, int c) {
    return (int64_t)op.uq * (uint32_t)c + (op.ur * (uint32_t)c) / (uint32_t)op.grid;
}

// Write this lane's outputs of one tile of output o (rows ra, rb local to it): c0 (row ra,
// col 2q), c1 (ra, 2q+1), c2 (rb, 2q), c3 (rb, 2q+1).
__device__ __forceinline__ void store_tile(const Op& op, int m, int o, int64_t ra, int64_t rb,
                                           int q, const float (&v)[4]) {
    const int c0 = 2 * q, c1 = 2 * q + 1;
    uint16_t* const y = op.y[o];
    const int64_t ldy = op.ldy[o], n = op.n[o];
    if (c0 < m) {
        if (ra < n) y[c0 * ldy + ra] = f2bf(v[0]);
        if (rb < n) y[c0 * ldy + rb] = f2bf(v[2]);
    }
    if (c1 < m) {
        if (ra < n) y[c1 * ldy + ra] = f2bf(v[1]);
        if (rb < n) y[c1 * ldy + rb] = f2bf(v[3]);
    }
}

// The epilogue of row group rg from its finished fp32 sums.
template <bool DUAL, bool MULTIO>
__device__ __forceinline__ void epilogue(const Op& op, int m, int64_t rg, int warp, int q,
                                         int pr_a, int pr_b, const float (&tot)[DUAL ? 2 : 1][4]) {
    const int o = MULTIO ? output_of(op, rg) : 0;
    const int64_t row0 = (rg - (o > 0 ? op.gend[o - 1] : 0)) * kRows + warp * 16;
    float v[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        if constexpr (DUAL) {
            const float a = tot[0][e] * op.g[0];
            const float b = tot[1][e] * op.g[1];
            v[e] = a / (1.0f + expf(-a)) * b;
        } else {
            v[e] = tot[0][e] * op.g[o];
        }
    }
    store_tile(op, m, o, row0 + pr_a, row0 + pr_b, q, v);
}

// ------------------------------------------------------------------------------------------
// the kernel

struct RingPos {
    int slot;
    uint32_t phase;  // parity of the ring pass in progress
    int issued;      // entries issued (producer) so far
    int units;       // units issued (producer) so far
};

// Producer warp: the TMA boxes of this CTA's units of one operation, into the ring.
template <bool DUAL, bool MULTIO, class LP>
__device__ __forceinline__ void produce_op(const LP& L, const Op& op, uint8_t* ring,
                                           uint64_t* full, uint64_t* empty, uint64_t* xreq,
                                           RingPos& r, bool& ok, uint64_t pol, int cta, int lane) {
    if (cta >= op.grid) return;
    const int64_t ub = range_begin(op, cta), ue = range_begin(op, cta + 1);
    const int ku = op.ku;
    int64_t rg = (uint32_t)ub / (uint32_t)ku;  // units < 2^31
    int b = (int)(ub - rg * ku);
    // output of row group rg and its first row group (a multi-output operation's outputs follow
    // one another; the dual's two streams share one output)
    int o = MULTIO ? output_of(op, rg) : 0;
    int64_t gbase = o > 0 ? op.gend[o - 1] : 0;
    const int S = L.slots;
    const int mode = op.scale_mode;
    const int64_t srow = op.k >> 4;
    for (int64_t u = ub; u < ue;) {
        if (r.units >= kPrefetch && r.units - (DUAL ? 1 : 2) < kPrefetch) {
            // the rest of the ring queues behind the consumers' first requests for x, which
            // would otherwise wait for every weight box issued before them
            if (lane == 0 && ok) ok = mbar_wait(xreq, 0);
            ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
        }
        if (ok && r.issued >= S) {
            if (lane == 0) ok = mbar_wait(&empty[r.slot], r.phase ^ 1u);
            ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
        }
        if (!ok) {
            if (lane == 0) atomicExch(L.error, 2);
            return;
        }
        // the entry's halves: the dual's two streams of unit u, or units u and u + 1
        const int halves = DUAL ? 2 : (ue - u >= 2 ? 2 : 1);
        uint8_t* const ent = ring + r.slot * kEntryBytes;
        if (lane == 0)
            mbar_expect_tx(&full[r.slot], halves * (mode == kScaleTma ? kSlotBytes : kWBytes));
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
            if (hf >= halves) break;
            uint8_t* dst = ent + hf * kSlotBytes;
            const int y = (int)((rg - gbase) * kRows);  // first row of the unit in output o
            const int mi = op.map0 + 2 * (DUAL ? hf : o);
            if (lane == 0) {
                tma_load_2d(dst, &L.maps[mi], b * kWRowBytes, y, &full[r.slot], pol);
                if (mode == kScaleTma)
                    tma_load_2d(dst + kWBytes, &L.maps[mi + 1], b * kSRowBytes, y, &full[r.slot],
                                pol);
            }
            if (mode != kScaleTma) {
                // the 16 scale codes of each row for this unit (fewer in a ragged last unit)
                const uint8_t* sbase = op.s[o + (DUAL ? hf : 0)];
                for (int rr = lane; rr < kRows; rr += 32) {
                    const int64_t row = (int64_t)y + rr;
                    const bool vrow = row < op.n[o];
                    const uint8_t* src = sbase + (vrow ? row * srow : 0);
                    uint8_t* d = dst + kWBytes + rr * kSRowBytes;
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
            }
            if (!DUAL || hf == 1) {
                // next unit
                ++u;
                ++r.units;
                if (++b == ku) {
                    b = 0;
                    ++rg;
                    if (MULTIO && o + 1 < op.outs && rg == op.gend[o]) gbase = op.gend[o++];
                }
            }
        }
        if (mode != kScaleTma) {
            if (mode == kScaleAsync8) cp_async_arrive(&full[r.slot]);
            else mbar_arrive(&full[r.slot]);
        }
        if (++r.slot == S) {
            r.slot = 0;
            r.phase ^= 1u;
        }
        ++r.issued;
    }
}

// Consumer warps: one operation's units of this CTA, the row groups it completes written out.
template <bool DUAL, bool MULTIO, class LP>
__device__ __forceinline__ void consume_op(const LP& L, const Op& op, uint8_t* ring,
                                           uint64_t* full, uint64_t* empty, uint64_t* xreq,
                                           bool& xreq_sent, uint4* xsm, RingPos& cr, bool& ok,
                                           int* s_amax, float* s_descale, int* s_last, int cta,
                                           int tid) {
    constexpr int NS = DUAL ? 2 : 1;
    const int grid = op.grid;
    if (cta >= grid) return;
    const int lane = tid & 31, warp = tid >> 5;
    const int g = lane >> 2, q = lane & 3;
    const int m = L.m;
    const int S = L.slots;
    const int ku = op.ku;
    const int64_t units = op.units;
    const int64_t kdim = op.k;
    const uint16_t* const xg = op.x;
    const int64_t ldx = op.ldx;
    float* const partial = op.partial;
    uint32_t* const arrive = op.arrive;
    const int64_t u_begin = range_begin(op, cta);
    const int64_t u_end = range_begin(op, cta + 1);
    const int64_t rg0 = (uint32_t)u_begin / (uint32_t)ku;  // units < 2^31
    const int b0 = (int)(u_begin - rg0 * ku);
    const int Lr = (int)(u_end - u_begin);
    const int uslots = Lr < ku ? Lr : ku;              // distinct 256-k units of the range
    const int xrow = 2 * uslots * kSlotU4 + kRowPadU4;  // uint4 per staged x row

    // x, y and the workspace may be produced / used by the preceding kernel: the first operation
    // waits for it here, after its set-up above
    if (!xreq_sent) pdl_wait();
    // an operation reading an earlier one's result waits until all its row groups are written
    if (op.wait_idx >= 0) {
        if (tid == 0 && !wait_count(L.done + op.wait_idx, op.wait_target, L.wait_ns))
            atomicExch(L.error, 4);  // results of this launch invalid
        named_barrier(1, kConsumers);
    }

    // stage x (raw bf16) for the range's units (two 128-k blocks each, mod ku) with cp.async;
    // chunk (q, j) of a block-row holds k = blk*128 + 32q + 8j .. +8, stored at position
    // 4q + (j ^ q) so that the four lanes of a row read distinct banks
    const int kblocks = (int)((kdim + kBlockK - 1) / kBlockK);
    const int per_row = 2 * uslots * kSlotU4;
    for (int mm = 0; mm < m; ++mm)
        for (int c = tid; c < per_row; c += kConsumers) {
            const int xslot = c >> 4, qq = (c >> 2) & 3, jj = c & 3;
            int ub = b0 + (xslot >> 1);
            if (ub >= ku) ub -= ku;
            const int blk = 2 * ub + (xslot & 1);
            const int64_t kk = (int64_t)blk * kBlockK + 32 * qq + 8 * jj;
            const bool valid = blk < kblocks && kk < kdim;
            cp_async16(&xsm[mm * xrow + xslot * kSlotU4 + qq * 4 + (jj ^ qq)],
                       xg + (valid ? mm * ldx + kk : 0), valid);
        }
    asm volatile("cp.async.commit_group;" ::: "memory");
    if (!xreq_sent) {
        named_barrier(1, kConsumers);      // every consumer has issued its copies of x ...
        if (tid == 0) mbar_arrive(xreq);   // ... so the producer may queue the rest of the ring
        xreq_sent = true;
    }
    asm volatile("cp.async.wait_group 0;" ::: "memory");
    named_barrier(1, kConsumers);
    {
        // per-row largest magnitude, then conversion in place to f16 * 2^e(m): row r belongs
        // to the kConsumerWarps / mp warps w with w / (kConsumerWarps / mp) == r (mp = M
        // rounded up to a power of two), which share its amax through shared memory only
        // when there is more than one of them
        const int mp = m <= 1 ? 1 : (m <= 2 ? 2 : (m <= 4 ? 4 : 8));
        const int wpr = kConsumerWarps / mp;
        const int r = warp / wpr, part = warp - r * wpr;
        uint32_t a = 0;
        if (r < m)
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
            if (lane == 0 && r < m) atomicMax(&s_amax[r], (int)a);
            named_barrier(1, kConsumers);
            a = r < m ? (uint32_t)s_amax[r] : 0u;
        }
        // a is the bf16 magnitude bit pattern of the row's largest |x| in the range; the scale
        // 2^e puts that maximum in [2^14, 2^15), inside f16's range
        int e = 0;
        if (a != 0u && a < 0x7F80u) e = 14 - ((int)(a >> 7) - 127);
        e = e > 126 ? 126 : (e < -126 ? -126 : e);
        const float sc = __uint_as_float((uint32_t)(e + 127) << 23);
        if (r < m) {
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
    const float ds0 = 2 * q < m ? s_descale[2 * q] : 1.f;
    const float ds1 = 2 * q + 1 < m ? s_descale[2 * q + 1] : 1.f;
    if (tid < 8) s_amax[tid] = 0;  // for the next operation (read again only after a barrier)

    // this lane's weight rows inside a tile (fragment rows g and g+8)
    const int pr_a = perm_row(g), pr_b = perm_row(g + 8);
    // this lane's x row: the mma's column g.  Columns g >= M are computed from row 0 and never
    // stored (partial tiles and outputs keep columns < M only), so the loads need no predicate.
    const uint4* const xrow_g = xsm + (g < m ? g : 0) * xrow + q * 4;
    const int frag = (warp * 32 + lane) * 4;  // this lane's floats in a partial tile

    float acc[NS][2][4];
#pragma unroll
    for (int s = 0; s < NS; ++s)
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[s][h][i] = 0.f;

    int finished = 0;
    int64_t cur_rg = rg0;
    int cur_b = b0, seg_b0 = b0;

    int ent = 0;  // ring entry of the current unit
#pragma unroll 1
    for (int i = 0; i < Lr; ++i) {
        int uslot = cur_b - b0;
        if (uslot < 0) uslot += ku;
        // an entry holds the dual's two streams of one unit, or two consecutive units
        const bool first_of_entry = DUAL || (i & 1) == 0;
        const bool last_of_entry = DUAL || (i & 1) == 1 || i + 1 == Lr;
        if (first_of_entry) {
            ent = cr.slot;
            if (ok && !mbar_wait(&full[cr.slot], cr.phase)) {
                ok = false;
                atomicExch(L.error, 3);
            }
            if (++cr.slot == S) {
                cr.slot = 0;
                cr.phase ^= 1u;
            }
        }
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            // the unit's two 128-k blocks: chunks 4h .. 4h+3 of each 128-byte row
            uint4 xv[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) xv[j] = xrow_g[(2 * uslot + h) * kSlotU4 + (j ^ q)];
            uint4 wa[NS], wb[NS];
            uint32_t sa[NS], sb[NS];
#pragma unroll
            for (int s = 0; s < NS; ++s) {
                const uint8_t* stage = ring + ent * kEntryBytes + (DUAL ? s : (i & 1)) * kSlotBytes;
                const uint8_t* sstage = stage + kWBytes;
                const int ra = warp * 16 + pr_a, rb = warp * 16 + pr_b;
                wa[s] = *reinterpret_cast<const uint4*>(stage + swz(ra, 4 * h + q));
                wb[s] = *reinterpret_cast<const uint4*>(stage + swz(rb, 4 * h + q));
                sa[s] = *reinterpret_cast<const uint16_t*>(sstage + ra * kSRowBytes + 8 * h + 2 * q);
                sb[s] = *reinterpret_cast<const uint16_t*>(sstage + rb * kSRowBytes + 8 * h + 2 * q);
            }
            if (h == 1 && last_of_entry) {
                // one arrival per warp, once all its lanes' reads of the entry are done
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[ent]);
            }
#pragma unroll
            for (int s = 0; s < NS; ++s) compute_tile(acc[s], wa[s], wb[s], sa[s], sb[s], xv);
        }

        if (cur_b + 1 == ku || i + 1 == Lr) {
            // ---- end of a row-group segment: units seg_b0 .. cur_b of row group cur_rg
            float tot[NS][4];
#pragma unroll
            for (int s = 0; s < NS; ++s)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    tot[s][e] = (acc[s][0][e] + acc[s][1][e]) * ((e & 1) ? ds1 : ds0);
                    acc[s][0][e] = 0.f;
                    acc[s][1][e] = 0.f;
                }
            const bool head = seg_b0 > 0;        // the group began before this range
            const bool tail = cur_b + 1 != ku;   // the group continues after it
            if (!head && !tail) {
                epilogue<DUAL, MULTIO>(op, m, cur_rg, warp, q, pr_a, pr_b, tot);
                ++finished;
            } else {
                const int c0 = head ? cta_of(units, grid, cur_rg * ku) : cta;
                const int c1 = cta_of(units, grid, (cur_rg + 1) * ku - 1);
                const uint32_t helpers = (uint32_t)(c1 - c0);  // later CTAs of the group
                bool fin = false;       // this CTA finishes the group
                bool own_regs = true;   // ... with its own part still in registers
                if (head) {
                    // a later CTA of the group: publish the partial tile, then count it in; if
                    // the owner already stopped waiting and this is the last tile, finish here
                    if (2 * q < m) {
#pragma unroll
                        for (int s = 0; s < NS; ++s)
                            *reinterpret_cast<float4*>(partial + ((int64_t)cta * 2 * NS + s) * kPartialFloats + frag) =
                                make_float4(tot[s][0], tot[s][1], tot[s][2], tot[s][3]);
                    }
                    // the RMW's release orders every consumer's partial stores (ordered before
                    // it by the barrier) ahead of the count at GPU scope
                    named_barrier(1, kConsumers);
                    if (tid == 0) {
                        const uint32_t old = atom_add_acq_rel(arrive + c0, 1u);
                        s_last[0] = (old & kOwnerGone) && (old & ~kOwnerGone) + 1u == helpers;
                    }
                    named_barrier(1, kConsumers);
                    fin = s_last[0] != 0;
                } else {
                    // the owner: wait for the later CTAs' tiles, normally already there
                    if (tid == 0) {
                        const uint64_t t0 = global_ns();
                        bool all = false;
                        for (int it = 0; it < kSpinLimit; ++it) {
                            if ((ld_acquire(arrive + c0) & ~kOwnerGone) == helpers) {
                                all = true;
                                break;
                            }
                            if ((int64_t)(global_ns() - t0) > L.owner_wait_ns) break;
                            __nanosleep(32);
                        }
                        s_last[1] = all;
                    }
                    named_barrier(1, kConsumers);
                    fin = s_last[1] != 0;
                    if (!fin) {
                        // they are late (not resident): publish this tile too and leave the
                        // group to the last of them, unless they all arrived meanwhile
                        if (2 * q < m) {
#pragma unroll
                            for (int s = 0; s < NS; ++s)
                                *reinterpret_cast<float4*>(partial + (((int64_t)cta * 2 + 1) * NS + s) * kPartialFloats + frag) =
                                    make_float4(tot[s][0], tot[s][1], tot[s][2], tot[s][3]);
                        }
                        named_barrier(1, kConsumers);
                        if (tid == 0) s_last[2] = (atom_or_acq_rel(arrive + c0, kOwnerGone) & ~kOwnerGone) == helpers;
                        named_barrier(1, kConsumers);
                        fin = s_last[2] != 0;
                    }
                }
                if (fin) {
                    // every CTA's tile in CTA order: the owner's tail, then the later CTAs' heads
                    float sum[NS][4];
#pragma unroll
                    for (int s = 0; s < NS; ++s)
#pragma unroll
                        for (int e = 0; e < 4; ++e) sum[s][e] = 0.f;
                    if (2 * q < m) {
                        for (int c = c0; c <= c1; ++c)
#pragma unroll
                            for (int s = 0; s < NS; ++s) {
                                const float4 v = (own_regs && c == cta)
                                    ? make_float4(tot[s][0], tot[s][1], tot[s][2], tot[s][3])
                                    : ld_cg4(partial + (((int64_t)c * 2 + (c == c0 ? 1 : 0)) * NS + s) * kPartialFloats + frag);
                                if (c == c0) {
                                    sum[s][0] = v.x;
                                    sum[s][1] = v.y;
                                    sum[s][2] = v.z;
                                    sum[s][3] = v.w;
                                } else {
                                    sum[s][0] += v.x;
                                    sum[s][1] += v.y;
                                    sum[s][2] += v.z;
                                    sum[s][3] += v.w;
                                }
                            }
                    }
                    epilogue<DUAL, MULTIO>(op, m, cur_rg, warp, q, pr_a, pr_b, sum);
                    if (tid == 0) arrive[c0] = 0u;  // the group is done: ready for the next launch
                    ++finished;
                }
            }
            seg_b0 = 0;
        }
        if (++cur_b == ku) {
            cur_b = 0;
            ++cur_rg;
        }
    }

    named_barrier(1, kConsumers);  // every read of this operation's staged x is done
    if (op.sig_idx >= 0) {
        // every finished group's output stores precede the release below
        named_barrier(1, kConsumers);
        if (tid == 0 && finished > 0) red_release_add(L.done + op.sig_idx, (uint32_t)finished);
    }
}

template <int MODE>
__global__ void __launch_bounds__(kThreads, 1)
    nvfp4_gemv_kernel(const __grid_constant__ LaunchOf<MODE> L) {
    extern __shared__ __align__(16) uint8_t smem_raw[];
    // the ring starts on a 1024-byte boundary (the launch reserves the slack)
    uint8_t* const ring = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint4* const xsm = reinterpret_cast<uint4*>(ring + L.slots * kEntryBytes);
    __shared__ __align__(8) uint64_t full_bar[kMaxSlots], empty_bar[kMaxSlots], xreq_bar;
    __shared__ int s_amax[8];
    __shared__ float s_descale[8];
    __shared__ int s_last[3];
    // a chain's operations are indexed at run time: each side works from a copy of its current
    // operation in shared memory ([0] the producer's, [1] the consumers'); the other modes read
    // operation 0 straight from the parameter bank
    __shared__ __align__(16) Op s_op[MODE == kModeChain ? 2 : 1];
    constexpr int kOpWords = sizeof(Op) / 4;
    static_assert(sizeof(Op) % 4 == 0, "operations are copied as words");

    pdl_launch_dependents();
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int cta = blockIdx.x;

    if (tid == 0) {
        for (int i = 0; i < kMaxSlots; ++i) {
            mbar_init(&full_bar[i], (uint32_t)L.full_count);
            mbar_init(&empty_bar[i], kConsumerWarps);
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
        const uint64_t pol = evict_first_policy();
        RingPos r{0, 0u, 0, 0};
        bool ok = true;
        for (int i = 0; i < L.ops && ok; ++i) {
            if constexpr (MODE == kModeSingle) {
                produce_op<false, false>(L, L.op[0], ring, full_bar, empty_bar, &xreq_bar, r, ok, pol, cta, lane);
            } else if constexpr (MODE == kModeDual) {
                produce_op<true, false>(L, L.op[0], ring, full_bar, empty_bar, &xreq_bar, r, ok, pol, cta, lane);
            } else if constexpr (MODE == kModeMulti) {
                produce_op<false, true>(L, L.op[0], ring, full_bar, empty_bar, &xreq_bar, r, ok, pol, cta, lane);
            } else {
                const uint32_t* src = reinterpret_cast<const uint32_t*>(&L.op[i]);
                for (int w = lane; w < kOpWords; w += 32) reinterpret_cast<uint32_t*>(&s_op[0])[w] = src[w];
                __syncwarp();
                const Op& op = s_op[0];
                const int lc = cta + op.rot < (int)gridDim.x ? cta + op.rot : cta + op.rot - (int)gridDim.x;
                if (op.dual)
                    produce_op<true, false>(L, op, ring, full_bar, empty_bar, &xreq_bar, r, ok, pol, lc, lane);
                else
                    produce_op<false, true>(L, op, ring, full_bar, empty_bar, &xreq_bar, r, ok, pol, lc, lane);
                __syncwarp();  // every lane is done with this copy
            }
        }
        asm volatile("cp.async.wait_all;" ::: "memory");
        return;
    }

    // ---- consumers ------------------------------------------------------------------------
    RingPos cr{0, 0u, 0, 0};
    bool ok = true, xreq_sent = false;
    for (int i = 0; i < L.ops; ++i) {
        if constexpr (MODE == kModeSingle) {
            consume_op<false, false>(L, L.op[0], ring, full_bar, empty_bar, &xreq_bar, xreq_sent, xsm, cr, ok, s_amax, s_descale, s_last, cta, tid);
        } else if constexpr (MODE == kModeDual) {
            consume_op<true, false>(L, L.op[0], ring, full_bar, empty_bar, &xreq_bar, xreq_sent, xsm, cr, ok, s_amax, s_descale, s_last, cta, tid);
        } else if constexpr (MODE == kModeMulti) {
            consume_op<false, true>(L, L.op[0], ring, full_bar, empty_bar, &xreq_bar, xreq_sent, xsm, cr, ok, s_amax, s_descale, s_last, cta, tid);
        } else {
            named_barrier(1, kConsumers);  // every consumer is done with the previous copy
            const uint32_t* src = reinterpret_cast<const uint32_t*>(&L.op[i]);
            for (int w = tid; w < kOpWords; w += kConsumers) reinterpret_cast<uint32_t*>(&s_op[1])[w] = src[w];
            named_barrier(1, kConsumers);
            const Op& op = s_op[1];
            const int lc = cta + op.rot < (int)gridDim.x ? cta + op.rot : cta + op.rot - (int)gridDim.x;
            if (op.dual)
                consume_op<true, false>(L, op, ring, full_bar, empty_bar, &xreq_bar, xreq_sent, xsm, cr, ok, s_amax, s_descale, s_last, lc, tid);
            else
                consume_op<false, true>(L, op, ring, full_bar, empty_bar, &xreq_bar, xreq_sent, xsm, cr, ok, s_amax, s_descale, s_last, lc, tid);
        }
    }
    if (!xreq_sent) pdl_wait();  // a CTA without units in any operation
    if (L.signals && tid == 0) {
        // the last CTA out (every CTA has passed all of its waits) clears the completion
        // counts for the next launch
        const uint32_t old = atom_add_acq_rel(L.exit_count, 1u);
        if (old + 1u == gridDim.x) {
            for (int i = 0; i < kMaxChainOps; ++i) L.done[i] = 0u;
            *L.exit_count = 0u;
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

bool g_attr_set[4][64];  // per kernel mode and device

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

// Bytes of one kernel operation's hand-off words and partial tiles.
size_t arrive_bytes(int sms) { return align_up((size_t)sms * 4, 256); }
size_t partial_bytes(int sms, int streams) {
    return (size_t)sms * 2 * streams * kPartialFloats * sizeof(float);
}

// Workspace of a single call: the header, then one operation's hand-off words and partial tiles
// (sized for two streams, so that every kind of call fits).
size_t workspace_layout(int sms, size_t* arrive_off, size_t* partial_off) {
    *arrive_off = kHeaderBytes;
    *partial_off = kHeaderBytes + arrive_bytes(sms);
    return *partial_off + partial_bytes(sms, 2);
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
    if (n > (int64_t(1) << 31) - kRows) return NVFP4_ERR_SHAPE;
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

// One output of an operation: its weight streams (two for the dual, gate then up), their
// global scales, and its rows.
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
// fit shared memory beside the smallest ring (kMinStages units of `streams` slots).
int64_t max_groups_per_launch(int streams, int64_t k, int sms) {
    const int ku = (int)((k + kUnitK - 1) / kUnitK);
    const size_t mx = NVFP4_PASS_ROWS;
    const int64_t max_slots =
        (int64_t)((kSmemMax - 1024 - (size_t)kMinStages * streams * kSlotBytes -
                   mx * kRowPadU4 * 16) /
                  (mx * kXSlotBytes));
    if (max_slots >= ku) return -1;
    const int64_t groups = (int64_t)sms * max_slots / ku;
    return groups > 0 ? groups : 1;
}

// How the producer moves an operation's scale codes: TMA needs 16-byte aligned scale rows.
int scale_mode_of(const Span* sp, int count, int streams, int64_t k) {
    int mode = kScaleTma;
    for (int o = 0; o < count; ++o)
        for (int i = 0; i < streams; ++i)
            if ((k % kUnitK) != 0 || misaligned(sp[o].s[i], 16)) mode = kScaleAsync8;
    if (mode == kScaleAsync8) {
        for (int o = 0; o < count; ++o)
            for (int i = 0; i < streams; ++i)
                if ((k % kBlockK) != 0 || misaligned(sp[o].s[i], 8)) mode = kScaleScalar;
    }
    return mode;
}

// Fills one kernel operation over the spans' row groups (concatenated in order; the dual takes
// one span), encoding its tensor maps at maps[*nmaps..].  Its split is that of a launch of this
// operation alone.
int fill_op(Op& op, CUtensorMap* maps, int* nmaps, int max_maps, const Span* sp, int count,
            bool dual, const void* x, int64_t ldx, int64_t k, int scale_mode, int sms,
            uint32_t* arrive, float* partial) {
    const int NS = dual ? 2 : 1;
    if (*nmaps + 2 * NS * count > max_maps) return NVFP4_ERR_SHAPE;
    memset(&op, 0, sizeof(op));
    op.map0 = *nmaps;
    int64_t groups = 0;
    for (int o = 0; o < count; ++o) {
        const Span& a = sp[o];
        for (int i = 0; i < NS; ++i) {
            const int slot = dual ? i : o;  // map / pointer slot of output o or of stream i
            op.s[slot] = a.s[i];
            op.g[slot] = a.g[i];
            CUtensorMap* mw = &maps[op.map0 + 2 * slot];
            if (!encode_map(mw, a.w[i], a.n, k / 2, kWRowBytes, kRows, CU_TENSOR_MAP_SWIZZLE_128B))
                return NVFP4_ERR_LAUNCH;
            if (scale_mode == kScaleTma &&
                !encode_map(mw + 1, a.s[i], a.n, k / 16, kSRowBytes, kRows,
                            CU_TENSOR_MAP_SWIZZLE_NONE))
                return NVFP4_ERR_LAUNCH;
        }
        op.y[o] = static_cast<uint16_t*>(a.y);
        op.ldy[o] = a.ldy;
        op.n[o] = a.n;
        groups += (a.n + kRows - 1) / kRows;
        op.gend[o] = groups;
    }
    *nmaps += 2 * NS * count;
    op.outs = count;
    op.dual = dual ? 1 : 0;
    op.x = static_cast<const uint16_t*>(x);
    op.ldx = ldx;
    op.k = k;
    op.ku = (int)((k + kUnitK - 1) / kUnitK);
    op.units = groups * op.ku;
    op.grid = (int)(op.units < sms ? op.units : sms);
    op.uq = (uint32_t)(op.units / op.grid);
    op.ur = (uint32_t)(op.units % op.grid);
    op.scale_mode = scale_mode;
    op.wait_idx = -1;
    op.sig_idx = -1;
    op.arrive = arrive;
    op.partial = partial;
    return NVFP4_OK;
}

// Staged x bytes of an operation's largest range at m rows.
size_t op_x_bytes(const Op& op, int m) {
    const int64_t max_range = (op.units + op.grid - 1) / op.grid;
    const int slots = (int)(max_range < op.ku ? max_range : op.ku);
    return (size_t)m * ((size_t)slots * kXSlotBytes + kRowPadU4 * 16);
}

template <int MODE>
int launch_kernel(const LaunchOf<MODE>& L, int grid, size_t smem, bool pdl, bool coop,
                  cudaStream_t stream) {
    int dev = 0;
    DeviceInfo* di = nullptr;
    int st = device_info(&dev, &di);
    if (st != NVFP4_OK) return st;
    if (!g_attr_set[MODE][dev]) {
        if (cudaFuncSetAttribute(nvfp4_gemv_kernel<MODE>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemMax) !=
            cudaSuccess) {
            cudaGetLastError();
            return NVFP4_ERR_LAUNCH;
        }
        g_attr_set[MODE][dev] = true;
    }
    cudaLaunchConfig_t cfg;
    memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    int na = 0;
    if (pdl) {
        attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[na].val.programmaticStreamSerializationAllowed = 1;
        ++na;
    }
    if (coop) {
        attr[na].id = cudaLaunchAttributeCooperative;
        attr[na].val.cooperative = 1;
        ++na;
    }
    cfg.attrs = na ? attr : nullptr;
    cfg.numAttrs = na;
    if (cudaLaunchKernelEx(&cfg, nvfp4_gemv_kernel<MODE>, L) != cudaSuccess) {
        cudaGetLastError();
        return NVFP4_ERR_LAUNCH;
    }
    return NVFP4_OK;
}

// Ring slots that fit beside `xbytes` of staged x.
int ring_slots(size_t xbytes) {
    if (xbytes + 1024 >= (size_t)kSmemMax) return 0;
    int slots = (int)((kSmemMax - 1024 - xbytes) / kEntryBytes);
    return slots > kMaxSlots ? kMaxSlots : slots;
}

// One launch over the spans' row groups, concatenated in order (the dual takes one span; more
// than one span needs MULTI).
template <bool DUAL, bool MULTI>
int launch_spans(const Span* sp, int count, const void* x, int64_t ldx, int m, int64_t k,
                 void* ws, size_t ws_bytes, uint32_t flags, cudaStream_t stream) {
    static_assert(!(DUAL && MULTI), "the dual kernel has one output");
    constexpr int MODE = DUAL ? kModeDual : (MULTI ? kModeMulti : kModeSingle);
    constexpr int NS = DUAL ? 2 : 1;
    if (count > (DUAL ? 1 : (MULTI ? kMaxOutputs : 1))) return NVFP4_ERR_SHAPE;
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
    int dev = 0;
    DeviceInfo* di = nullptr;
    int st = device_info(&dev, &di);
    if (st != NVFP4_OK) return st;
    size_t arrive_off, partial_off;
    const size_t need = workspace_layout(di->sms, &arrive_off, &partial_off);
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

    LaunchOf<MODE> L;
    memset(&L, 0, sizeof(L));
    char* wsb = static_cast<char*>(ws);
    int nmaps = 0;
    const int scale_mode = scale_mode_of(sp, count, NS, k);
    if ((st = fill_op(L.op[0], L.maps, &nmaps, ModeCfg<MODE>::kMaps, sp, count, DUAL, x, ldx, k,
                      scale_mode, di->sms, reinterpret_cast<uint32_t*>(wsb + arrive_off),
                      reinterpret_cast<float*>(wsb + partial_off))) != NVFP4_OK)
        return st;
    L.ops = 1;
    L.m = m;
    L.full_count = scale_mode == kScaleTma ? 1 : 1 + 32;
    L.signals = 0;
    L.wait_ns = kDefaultWaitNs;
    L.owner_wait_ns = kOwnerWaitNs;
    L.done = reinterpret_cast<uint32_t*>(wsb + kDoneOffset);
    L.exit_count = reinterpret_cast<uint32_t*>(wsb + 4);
    L.error = reinterpret_cast<int32_t*>(wsb);
    const size_t xbytes = op_x_bytes(L.op[0], m);
    L.slots = ring_slots(xbytes);
    if (L.slots * 2 < kMinStages * NS) return NVFP4_ERR_LAUNCH;  // cannot happen: the split bounds x
    const size_t smem = 1024 + (size_t)L.slots * kEntryBytes + xbytes;
    return launch_kernel<MODE>(L, L.op[0].grid, smem, (flags & NVFP4_FLAG_PREFETCH_WEIGHTS) != 0,
                               false, stream);
}

// One output (one or two weight streams), split into launches of at most
// max_groups_per_launch row groups.
template <bool DUAL>
int launch(const uint8_t* const* w, const uint8_t* const* s, const float* gs, const void* x,
           int64_t ldx, void* y, int64_t ldy, int m, int64_t n, int64_t k, void* ws,
           size_t ws_bytes, uint32_t flags, cudaStream_t stream) {
    constexpr int NS = DUAL ? 2 : 1;
    int dev = 0;
    DeviceInfo* di = nullptr;
    int st = device_info(&dev, &di);
    if (st != NVFP4_OK) return st;
    const int64_t cap = max_groups_per_launch(NS, k, di->sms);
    const int64_t rows_per_launch = cap < 0 ? n : cap * kRows;
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
    size_t arrive_off, partial_off;
    const size_t base = workspace_layout(di->sms, &arrive_off, &partial_off);
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

// ------------------------------------------------------------------------------------------
// chains

// A chain's operation as the kernel runs it: the caller's operation i, or one row chunk of it
// when its row groups exceed one launch's limit at its K (split as nvfp4_gemv splits them).
struct ChainPiece {
    Span sp[kMaxOutputs];
    int count;
    bool dual;
    int src;       // the caller's operation
    int64_t k;
};

// Checks a chain and cuts it into the kernel's operations.  x of each piece is resolved by the
// caller of this function per 8-row pass.  With sms == 0 it only checks the arguments (no CUDA
// call needed).
int plan_chain(const nvfp4_chain_op_t* ops, int count, int m, int sms, ChainPiece* pieces,
               int* npieces, int64_t* groups_of) {
    if (!ops) return NVFP4_ERR_NULL;
    if (count < 1 || count > kMaxChainOps) return NVFP4_ERR_SHAPE;
    if (m < 1 || m > NVFP4_MAX_ROWS) return NVFP4_ERR_ROWS;
    int np = 0;
    for (int i = 0; i < count; ++i) {
        const nvfp4_chain_op_t& a = ops[i];
        const bool dual = a.kind == NVFP4_OP_DUAL;
        if (!dual && a.kind != NVFP4_OP_SINGLE) return NVFP4_ERR_SHAPE;
        const int outs = dual ? 1 : a.outputs;
        if (outs < 1 || outs > kMaxOutputs || (dual && a.outputs != 1)) return NVFP4_ERR_SHAPE;
        const int64_t k = a.k;
        if (k <= 0 || (k % kUnitK) != 0 || k > kMaxK) return NVFP4_ERR_SHAPE;
        if (a.x_from >= i || a.x_from < -1) return NVFP4_ERR_SHAPE;
        if (a.x_from >= 0) {
            const nvfp4_chain_op_t& src = ops[a.x_from];
            const int src_outs = src.kind == NVFP4_OP_DUAL ? 1 : src.outputs;
            if (src_outs != 1 || src.out[0].n != k) return NVFP4_ERR_SHAPE;
            if ((src.out[0].ldy % 8) != 0 || misaligned(src.out[0].y, 16)) return NVFP4_ERR_ALIGN;
        } else {
            if (!a.x) return NVFP4_ERR_NULL;
            if (a.ldx < k) return NVFP4_ERR_SHAPE;
            if ((a.ldx % 8) != 0 || misaligned(a.x, 16)) return NVFP4_ERR_ALIGN;
        }
        const int NS = dual ? 2 : 1;
        Span sp[kMaxOutputs];
        memset(sp, 0, sizeof(sp));
        int64_t groups = 0;
        for (int o = 0; o < outs; ++o) {
            const nvfp4_output_t& b = a.out[o];
            if (b.n <= 0 || b.n > (int64_t(1) << 31) - kRows) return NVFP4_ERR_SHAPE;
            if (b.ldy < b.n) return NVFP4_ERR_SHAPE;
            if (!b.y) return NVFP4_ERR_NULL;
            if (misaligned(b.y, 2)) return NVFP4_ERR_ALIGN;
            int st = check_weight(b.w, b.s);
            if (st != NVFP4_OK) return st;
            if (misaligned(b.s, 16)) return NVFP4_ERR_ALIGN;  // scale boxes by TMA
            sp[o].w[0] = b.w;
            sp[o].s[0] = b.s;
            sp[o].g[0] = b.global_scale;
            sp[o].y = b.y;
            sp[o].ldy = b.ldy;
            sp[o].n = b.n;
            groups += (b.n + kRows - 1) / kRows;
        }
        if (dual) {
            const nvfp4_output_t& u = a.out[1];
            if (u.n != a.out[0].n) return NVFP4_ERR_SHAPE;
            int st = check_weight(u.w, u.s);
            if (st != NVFP4_OK) return st;
            if (misaligned(u.s, 16)) return NVFP4_ERR_ALIGN;
            sp[0].w[1] = u.w;
            sp[0].s[1] = u.s;
            sp[0].g[1] = u.global_scale;
        }
        groups_of[i] = groups;
        const int64_t cap = sms > 0 ? max_groups_per_launch(NS, k, sms) : -1;
        if (cap < 0 || groups <= cap) {
            if (np == kMaxChainOps) return NVFP4_ERR_SHAPE;
            ChainPiece& p = pieces[np++];
            memcpy(p.sp, sp, sizeof(sp));
            p.count = outs;
            p.dual = dual;
            p.src = i;
            p.k = k;
            continue;
        }
        // too many row groups for one launch at this K: each output in row chunks, as
        // nvfp4_gemv and nvfp4_gemv_multi run them
        const int64_t rows_per = cap * kRows;
        for (int o = 0; o < outs; ++o)
            for (int64_t r0 = 0; r0 < sp[o].n; r0 += rows_per) {
                if (np == kMaxChainOps) return NVFP4_ERR_SHAPE;
                ChainPiece& p = pieces[np++];
                memset(&p, 0, sizeof(p));
                for (int s = 0; s < NS; ++s) {
                    p.sp[0].w[s] = sp[o].w[s] + r0 * (k / 2);
                    p.sp[0].s[s] = sp[o].s[s] + r0 * (k / 16);
                    p.sp[0].g[s] = sp[o].g[s];
                }
                p.sp[0].y = static_cast<uint16_t*>(sp[o].y) + r0;
                p.sp[0].ldy = sp[o].ldy;
                p.sp[0].n = sp[o].n - r0 < rows_per ? sp[o].n - r0 : rows_per;
                p.count = 1;
                p.dual = dual;
                p.src = i;
                p.k = k;
            }
    }
    *npieces = np;
    return NVFP4_OK;
}

// Workspace bytes of a chain cut into these pieces.
size_t chain_layout(const ChainPiece* pieces, int np, int sms, size_t* off) {
    size_t at = kHeaderBytes;
    for (int i = 0; i < np; ++i) {
        off[i] = at;
        at += arrive_bytes(sms) + partial_bytes(sms, pieces[i].dual ? 2 : 1);
    }
    return at;
}

// One 8-row pass of a chain (rows r0 .. r0 + m - 1 of every x and y).
int launch_chain_pass(const nvfp4_chain_op_t* ops, int count, const ChainPiece* pieces, int np,
                      const int64_t* groups_of, int r0, int m, int sms, void* ws,
                      const size_t* off, uint32_t flags, int64_t wait_ns, int unsignalled,
                      int64_t owner_wait_ns,
                      cudaStream_t stream) {
    // LaunchOf<kModeChain> is about 13 KB: keep it off the stack of small host threads
    static thread_local LaunchOf<kModeChain> L;
    memset(&L, 0, sizeof(L));
    char* wsb = static_cast<char*>(ws);
    bool read[kMaxChainOps] = {false};  // the caller's operations whose result a later one reads
    for (int i = 0; i < count; ++i)
        if (ops[i].x_from >= 0) read[ops[i].x_from] = true;
    // the test form leaves the first operation that another one reads unsignalled
    int first_read = -1;
    for (int i = count - 1; i >= 0; --i)
        if (read[i]) first_read = i;
    int nmaps = 0;
    size_t xmax = 0;
    bool waits = false;
    for (int p = 0; p < np; ++p) {
        const ChainPiece& c = pieces[p];
        const nvfp4_chain_op_t& a = ops[c.src];
        Span sp[kMaxOutputs];
        for (int o = 0; o < c.count; ++o) {
            sp[o] = c.sp[o];
            sp[o].y = static_cast<uint16_t*>(c.sp[o].y) + (int64_t)r0 * c.sp[o].ldy;
        }
        const void* x;
        int64_t ldx;
        if (a.x_from >= 0) {
            const nvfp4_output_t& src = ops[a.x_from].out[0];
            x = static_cast<const uint16_t*>(src.y) + (int64_t)r0 * src.ldy;
            ldx = src.ldy;
        } else {
            x = static_cast<const uint16_t*>(a.x) + (int64_t)r0 * a.ldx;
            ldx = a.ldx;
        }
        Op& op = L.op[p];
        int st = fill_op(op, L.maps, &nmaps, kChainMaps, sp, c.count, c.dual, x, ldx, c.k,
                         kScaleTma, sms, reinterpret_cast<uint32_t*>(wsb + off[p]),
                         reinterpret_cast<float*>(wsb + off[p] + arrive_bytes(sms)));
        if (st != NVFP4_OK) return st;
        if (a.x_from >= 0) {
            op.wait_idx = a.x_from;
            op.wait_target = (uint32_t)groups_of[a.x_from];
            waits = true;
        }
        if (read[c.src] && !(unsignalled && c.src == first_read)) op.sig_idx = c.src;
        op.rot = p % sms;
        const size_t xb = op_x_bytes(op, m);
        if (xb > xmax) xmax = xb;
    }
    L.ops = np;
    L.m = m;
    L.full_count = 1;
    L.signals = waits ? 1 : 0;
    L.wait_ns = wait_ns;
    L.owner_wait_ns = owner_wait_ns;
    L.done = reinterpret_cast<uint32_t*>(wsb + kDoneOffset);
    L.exit_count = reinterpret_cast<uint32_t*>(wsb + 4);
    L.error = reinterpret_cast<int32_t*>(wsb);
    L.slots = ring_slots(xmax);
    if (L.slots < 2) return NVFP4_ERR_SHAPE;
    const size_t smem = 1024 + (size_t)L.slots * kEntryBytes + xmax;
    // every CTA runs every operation; a chain with waits needs all of them resident at once
    return launch_kernel<kModeChain>(L, sms, smem, (flags & NVFP4_FLAG_PREFETCH_WEIGHTS) != 0,
                                     waits, stream);
}

int run_chain(const nvfp4_chain_op_t* ops, int count, int m, void* ws, size_t ws_bytes,
              uint32_t flags, int64_t wait_ns, int unsignalled, int64_t owner_wait_ns,
              cudaStream_t stream) {
    if (flags & ~(uint32_t)NVFP4_FLAG_PREFETCH_WEIGHTS) return NVFP4_ERR_SHAPE;
    ChainPiece pieces[kMaxChainOps];
    int np = 0;
    int64_t groups_of[kMaxChainOps];
    int st = plan_chain(ops, count, m, 0, pieces, &np, groups_of);
    if (st != NVFP4_OK) return st;
    if (!ws || misaligned(ws, 16)) return NVFP4_ERR_WORKSPACE;
    int dev = 0;
    DeviceInfo* di = nullptr;
    if ((st = device_info(&dev, &di)) != NVFP4_OK) return st;
    if ((st = plan_chain(ops, count, m, di->sms, pieces, &np, groups_of)) != NVFP4_OK) return st;
    size_t off[kMaxChainOps];
    if (!ws || misaligned(ws, 16) || ws_bytes < chain_layout(pieces, np, di->sms, off))
        return NVFP4_ERR_WORKSPACE;
    for (int r0 = 0; r0 < m; r0 += NVFP4_PASS_ROWS) {
        const int rows = m - r0 < NVFP4_PASS_ROWS ? m - r0 : NVFP4_PASS_ROWS;
        if ((st = launch_chain_pass(ops, count, pieces, np, groups_of, r0, rows, di->sms, ws, off,
                                    flags, wait_ns, unsignalled, owner_wait_ns, stream)) != NVFP4_OK)
            return st;
    }
    return NVFP4_OK;
}

}  // namespace

// ------------------------------------------------------------------------------------------
// Scratch of nvfp4_gemv_noalloc: the workspace of nvfp4_gemv (header, one hand-off word per CTA,
// two pairs of partial tiles per CTA, in workspace_layout's order) compiled into the library
// for grids of up to kNoAllocSms CTAs, so that the call needs no buffer from its caller.

constexpr int kNoAllocSms = 160;
constexpr size_t kNoAllocArriveBytes = ((size_t)kNoAllocSms * 4 + 255) / 256 * 256;
constexpr size_t kNoAllocBytes = kHeaderBytes + kNoAllocArriveBytes +
                                 (size_t)kNoAllocSms * 2 * 2 * kPartialFloats * sizeof(float);
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocBytes];

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
        size_t arrive_off, partial_off;
        const size_t base = workspace_layout(di->sms, &arrive_off, &partial_off);
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
    size_t arrive_off, partial_off;
    if (workspace_layout(di->sms, &arrive_off, &partial_off) > kNoAllocBytes)
        return NVFP4_ERR_WORKSPACE;  // more SMs than the compiled-in scratch covers
    // The array's device address in the current context, looked up on every call (a host-side
    // table lookup, no allocation), so that it stays right after a context is recreated.
    void* scratch = nullptr;
    if (cudaGetSymbolAddress(&scratch, g_noalloc_scratch) != cudaSuccess || !scratch) {
        cudaGetLastError();
        return NVFP4_ERR_LAUNCH;
    }
    // The previous call left its error word and counts behind; start this one from zero.
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
        size_t arrive_off, partial_off;
        const size_t base = workspace_layout(di->sms, &arrive_off, &partial_off);
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
            size_t arrive_off, partial_off;
            const size_t base = workspace_layout(di->sms, &arrive_off, &partial_off);
            return nvfp4_tc::launch_multi(g_encode, di->sms, tw, ts, tg, ty, tldy, tn, used, x,
                                          ldx, m, k, pro, workspace, workspace_bytes, base,
                                          stream);
        }
    }
    if ((st = prologue_pass(pro, &x, &ldx, m, k, workspace, workspace_bytes, flags, stream)) !=
        NVFP4_OK)
        return st;
    int64_t groups = 0;
    for (int o = 0; o < used; ++o) groups += (sp[o].n + kRows - 1) / kRows;
    const int64_t cap = max_groups_per_launch(1, k, di->sms);
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

int nvfp4_chain_workspace_bytes(const nvfp4_chain_op_t* ops, int count, int m, size_t* bytes) {
    if (!bytes) return NVFP4_ERR_NULL;
    ChainPiece pieces[kMaxChainOps];
    int np = 0;
    int64_t groups_of[kMaxChainOps];
    int st = plan_chain(ops, count, m, 0, pieces, &np, groups_of);
    if (st != NVFP4_OK) return st;
    int dev = 0;
    DeviceInfo* di = nullptr;
    if ((st = device_info(&dev, &di)) != NVFP4_OK) return st;
    if ((st = plan_chain(ops, count, m, di->sms, pieces, &np, groups_of)) != NVFP4_OK) return st;
    size_t off[kMaxChainOps];
    *bytes = chain_layout(pieces, np, di->sms, off);
    return NVFP4_OK;
}

int nvfp4_gemv_chain(const nvfp4_chain_op_t* ops, int count, int m, void* workspace,
                     size_t workspace_bytes, uint32_t flags, cudaStream_t stream) {
    return run_chain(ops, count, m, workspace, workspace_bytes, flags, kDefaultWaitNs, 0,
                     kOwnerWaitNs, stream);
}

int nvfp4_gemv_chain_unsignalled(const nvfp4_chain_op_t* ops, int count, int m, void* workspace,
                                 size_t workspace_bytes, int64_t wait_limit_ns,
                                 cudaStream_t stream) {
    if (wait_limit_ns <= 0 || wait_limit_ns > kDefaultWaitNs) return NVFP4_ERR_SHAPE;
    return run_chain(ops, count, m, workspace, workspace_bytes, 0u, wait_limit_ns, 1,
                     kOwnerWaitNs, stream);
}

int nvfp4_gemv_chain_owner_wait(const nvfp4_chain_op_t* ops, int count, int m, void* workspace,
                                size_t workspace_bytes, int64_t owner_wait_ns,
                                cudaStream_t stream) {
    if (owner_wait_ns < 0 || owner_wait_ns > kOwnerWaitNs) return NVFP4_ERR_SHAPE;
    return run_chain(ops, count, m, workspace, workspace_bytes, 0u, kDefaultWaitNs, 0,
                     owner_wait_ns, stream);
}

int nvfp4_workspace_bytes_wide(int64_t n, int64_t k, int m, size_t* bytes) {
    if (!bytes) return NVFP4_ERR_NULL;
    if (n < 0 || k < 0 || (k % 32) != 0 || k > kMaxK) return NVFP4_ERR_SHAPE;
    if (m < 0 || m > NVFP4_MAX_ROWS) return NVFP4_ERR_ROWS;
    int dev = 0;
    DeviceInfo* di = nullptr;
    int st = device_info(&dev, &di);
    if (st != NVFP4_OK) return st;
    size_t arrive_off, partial_off;
    const size_t tier = m > NVFP4_PASS_ROWS ? nvfp4_tc::scratch_bytes(n, k, m, di->sms) : 0;
    const size_t pro = prologue_scratch_bytes(m, k);
    *bytes = workspace_layout(di->sms, &arrive_off, &partial_off) + (tier > pro ? tier : pro);
    return NVFP4_OK;
}

int nvfp4_workspace_error(const void* workspace, size_t workspace_bytes, cudaStream_t stream,
                          int32_t* error) {
    if (!error) return NVFP4_ERR_NULL;
    if (!workspace || workspace_bytes < kHeaderBytes || misaligned(workspace, 16))
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
