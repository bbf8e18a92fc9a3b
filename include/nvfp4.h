/*
 * nvfp4.h -- C ABI of the weight-only NVFP4 GEMV library for NVIDIA B200 (sm_100a).
 *
 * The operation is the weight-only 4-bit GEMV of a decoder's decode step: the kernel family
 * the GB10 plan calls "w4a16_gemv" (w4a16_gemv_sw / w4a16_gemv_qg, single output) and
 * "w4a16_gemv_dual" (two weight streams sharing one activation), with weights in format
 * "nvfp4/g16" and bf16 activations ("Blueprint - circuit executor" page for
 * qwen3.8-27b-nvfp4 on GB10, tables "Kernels the plan launches" and "Weighted nodes").
 * Row counts 1 (plain decode) to 8 (an 8-row speculative draft/verify round, kern-qwen38-sm103
 * model card, section "Run"; NInfer card, DFlash2 "block width 8"), and up to 128 for the plan's
 * wider arms (multi_seq rows 2..128, same page, table "Plan arms").  One kernel pass computes
 * up to NVFP4_PASS_ROWS = 8 rows; a call with more rows runs ceil(M/8) passes over consecutive
 * 8-row blocks, each pass streaming the weights again (mostly from L2 when they fit there).
 *
 * Storage layout (layout_version 1):
 *   W  uint8 [N][K/2]   byte b of row n holds element k = 2b in bits 0..3 and k = 2b+1 in
 *                       bits 4..7; each element is E2M1 (sign bit 3, exponent bits 2..1 with
 *                       bias 1, mantissa bit 0; exponent 0 is subnormal 0.5*m).
 *   S  uint8 [N][K/16]  one E4M3 (FN variant, bias 7, max 448) scale per 16 elements along K,
 *                       row-major.  Scale codes must be non-negative finite (0x00..0x7E); the
 *                       sign bit and the NaN codes 0x7F/0xFF give unspecified results.
 *   g  float            per-tensor global scale, passed by value.
 *   x  bf16 [M][ldx]    activations, row-major, row stride ldx elements.
 *   y  bf16 [M][ldy]    outputs, row-major, row stride ldy elements.
 *
 *   y[m][n] = bf16_rn( g * sum_k E2M1(W[n][k]) * E4M3(S[n][k/16]) * x[m][k] )
 *
 * accumulated in fp32.  The fused dual computes, from two such weights sharing x,
 *   o[m][n] = bf16_rn( silu(g_gate * acc_gate) * (g_up * acc_up) ),  silu(t) = t / (1 + e^-t)
 * in fp32 -- the SiLU(gate)*up that the GB10 plan runs as a separate "moe_silu_mul" launch.
 *
 * Guarantees:
 *   - Row invariance: output row m is bitwise identical for every M in 1..128 given the same
 *     x row, weights, N, K and device (the kernel's work split depends on N, K and the SM
 *     count, never on M, and a row's arithmetic depends only on that row).
 *   - Determinism: identical calls give bitwise identical results.
 *
 * Conventions (every entry point):
 *   - Pointers are device pointers owned by the caller; the library never allocates, frees or
 *     synchronises.  Work is enqueued on `stream` and completes asynchronously; the buffers
 *     must stay valid until it has run.
 *   - Errors are returned as nvfp4_status codes (never exceptions or aborts).  Argument
 *     checks run on the host before any CUDA call.
 *   - The workspace (nvfp4_workspace_bytes) must be zero-filled before its first use.  It
 *     holds an error word, one hand-off word per CTA and fp32 partial sums: the persistent grid
 *     splits a weight's 128-row groups over the GPU's SMs, and a group cut between CTAs is
 *     finished by the CTA holding its first unit, which adds the others' partial sums in a fixed
 *     order.  That CTA waits for them at most 50 us; if they are not resident yet (other work
 *     holds SMs) it hands the group over and the last of them finishes it, so a call needs no
 *     co-residency of its CTAs and no wait is unbounded.  Every call that completes resets the
 *     words to zero, so the same workspace serves any number of calls in stream order (and
 *     CUDA-graph replays) without re-zeroing: the library is stateless per workspace, not per
 *     call.  Calls that may run concurrently (different streams) need different workspaces.
 */
#ifndef NVFP4_H
#define NVFP4_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* cudaStream_t;

typedef enum {
    NVFP4_OK = 0,
    NVFP4_ERR_NULL = -1,      /* a required pointer is NULL */
    NVFP4_ERR_SHAPE = -2,     /* N < 0, K < 0, K % 32 != 0, ldx < K, ldy < N, K too large */
    NVFP4_ERR_ROWS = -3,      /* M < 0 or M > NVFP4_MAX_ROWS (128) */
    NVFP4_ERR_ALIGN = -4,     /* pointer or stride alignment (see each call) */
    NVFP4_ERR_ARCH = -5,      /* current device is not compute capability 10.0 (B200) */
    NVFP4_ERR_LAUNCH = -6,    /* the CUDA launch failed (cudaGetLastError) */
    NVFP4_ERR_WORKSPACE = -7, /* workspace NULL, misaligned or smaller than required */
    NVFP4_ERR_ALIAS = -8      /* a prologue's residual output overlaps what the call reads or y */
} nvfp4_status;

#define NVFP4_MAX_ROWS 128 /* rows of x (and y) per call */
#define NVFP4_PASS_ROWS 8  /* rows one kernel pass computes; more run as ceil(M/8) passes */
#define NVFP4_MAX_OUTPUTS 4
#define NVFP4_GROUP 16
#define NVFP4_LAYOUT_VERSION 1

/* Flags of nvfp4_gemv_ex / nvfp4_gemv_dual_ex.
 * NVFP4_FLAG_PREFETCH_WEIGHTS: launch with programmatic dependent launch so that the packed
 *   weights and scales start streaming while the kernel enqueued before it on the stream is
 *   still running (the decode step's chain of projections overlaps one launch's tail with the
 *   next one's weight stream).  x, y and the workspace are still read and written only after
 *   that earlier work has completed.  Use it only when earlier work on the stream does not
 *   write the weights or scales of this call. */
#define NVFP4_FLAG_PREFETCH_WEIGHTS 1u
/* NVFP4_FLAG_WIDE_TENSOR (nvfp4_gemv_ex, nvfp4_gemv_dual_ex, nvfp4_gemv_multi and their _pro
 *   forms): calls of 9..128 rows with K % 256 == 0 and 16-byte aligned scale codes (every
 *   output's, for nvfp4_gemv_multi) run on the tensor-core tier instead of 8-row passes: one
 *   pass over each weight, tcgen05 MMAs on f16 operands (x carried with a power-of-two scale
 *   per row) with fp32 accumulation in tensor memory.  For nvfp4_gemv_dual_ex the gate and up
 *   results are kept in fp32 and combined by a final pass, o = bf16(silu(g_gate gate) *
 *   (g_up up)).  For nvfp4_gemv_multi x is converted once and each output is bitwise that of
 *   its own nvfp4_gemv_ex call with the flag.  Rows are then bitwise invariant for every M in
 *   9..128 and deterministic, and agree with calls of 1..8 rows within the stated tolerance
 *   (not bitwise).  The workspace must hold nvfp4_workspace_bytes_wide(N, K, M) bytes (for
 *   nvfp4_gemv_multi, the largest over its outputs).  Other calls ignore the flag. */
#define NVFP4_FLAG_WIDE_TENSOR 2u

typedef struct {
    int64_t n, k;
    int64_t weight_bytes;     /* N*K/2  */
    int64_t scale_bytes;      /* N*K/16 */
    int64_t weight_row_bytes; /* K/2    */
    int64_t scale_row_bytes;  /* K/16   */
    int32_t group;            /* 16 */
    int32_t max_rows;         /* 128 (NVFP4_MAX_ROWS) */
    int32_t align_bytes;      /* 16: required alignment of W and x */
    int32_t layout_version;   /* 1 */
} nvfp4_pack_info_t;

/* Sizes of the packed storage for an N x K weight (the "nvfp4/g16" format above).
 * Pure host function.  Returns NVFP4_ERR_NULL if out is NULL, NVFP4_ERR_SHAPE if
 * N < 0, K < 0 or K % 32 != 0. */
int nvfp4_pack_info(int64_t n, int64_t k, nvfp4_pack_info_t* out);

/* Bytes of workspace every GEMV call on the current device needs (depends only on the
 * device's SM count).  Returns NVFP4_ERR_NULL if bytes is NULL, NVFP4_ERR_ARCH if the current
 * device is not a B200 (no CUDA device included). */
int nvfp4_workspace_bytes(size_t* bytes);

/* y = W x (single output), see the header comment.
 *   w, x: 16-byte aligned;  s, y: 2-byte aligned;  workspace: 16-byte aligned, at least
 *   nvfp4_workspace_bytes() bytes, zero-filled before first use.
 *   ldx % 8 == 0, ldx >= K;  ldy >= N.  1 <= M <= 128 (M == 0 and N == 0 are no-ops);
 *   K % 32 == 0 (K == 0 writes zeros).
 * Enqueued on `stream`; returns NVFP4_OK or an nvfp4_status error (nothing is enqueued on
 * error). */
int nvfp4_gemv(const uint8_t* w, const uint8_t* s, float global_scale, const void* x,
               int64_t ldx, void* y, int64_t ldy, int m, int64_t n, int64_t k, void* workspace,
               size_t workspace_bytes, cudaStream_t stream);

/* o = silu(W_gate x) * (W_up x), fused (one pass over both weight streams), see the header
 * comment.  Gate and up are separate pointers with their own global scales; a stacked
 * [gate; up] buffer is passed as w_up = w_gate + N*K/2, s_up = s_gate + N*K/16.
 * Same alignment, shape and workspace rules as nvfp4_gemv. */
int nvfp4_gemv_dual(const uint8_t* w_gate, const uint8_t* s_gate, float global_gate,
                    const uint8_t* w_up, const uint8_t* s_up, float global_up, const void* x,
                    int64_t ldx, void* y, int64_t ldy, int m, int64_t n, int64_t k,
                    void* workspace, size_t workspace_bytes, cudaStream_t stream);

/* nvfp4_gemv / nvfp4_gemv_dual with launch flags (NVFP4_FLAG_*; unknown bits ->
 * NVFP4_ERR_SHAPE).  The plain entry points are these with flags = 0. */
int nvfp4_gemv_ex(const uint8_t* w, const uint8_t* s, float global_scale, const void* x,
                  int64_t ldx, void* y, int64_t ldy, int m, int64_t n, int64_t k,
                  void* workspace, size_t workspace_bytes, uint32_t flags, cudaStream_t stream);
int nvfp4_gemv_dual_ex(const uint8_t* w_gate, const uint8_t* s_gate, float global_gate,
                       const uint8_t* w_up, const uint8_t* s_up, float global_up, const void* x,
                       int64_t ldx, void* y, int64_t ldy, int m, int64_t n, int64_t k,
                       void* workspace, size_t workspace_bytes, uint32_t flags,
                       cudaStream_t stream);

/* One output of nvfp4_gemv_multi: an N x K weight in the format above, its global scale, and
 * where its N outputs go.  w: 16-byte aligned; s, y: 2-byte aligned; ldy >= n. */
typedef struct {
    const uint8_t* w;      /* packed weights [n][K/2] */
    const uint8_t* s;      /* scale codes [n][K/16] */
    float global_scale;
    void* y;               /* bf16 [M][ldy] */
    int64_t ldy;
    int64_t n;             /* rows of this weight; 0 skips the output */
} nvfp4_output_t;

/* Several single-output GEMVs that share x and K, in one pass: for every output o,
 *   y_o[m][n] = bf16_rn( g_o * sum_k E2M1(W_o[n][k]) * E4M3(S_o[n][k/16]) * x[m][k] ).
 * The decode plan runs such groups as one launch: the attention k and v projections (the GB10
 * plan's two-output "w4a16_gemv_dual", 16 launches per step) and the gated attention's q and gate
 * ("w4a16_gemv_qg") ("Blueprint - circuit executor" page, table "Kernels the plan launches").
 *   outputs: `count` (1..NVFP4_MAX_OUTPUTS) descriptors, host memory, read during the call only.
 *   x, ldx, m, k, workspace, flags, stream: as nvfp4_gemv_ex.
 * The row groups of all outputs form one stream-K split over the GPU, so one launch streams
 * every weight.  When K is so large that nvfp4_gemv itself would split an output's rows over
 * several launches, and the outputs together exceed one launch, each output runs as its own
 * nvfp4_gemv_ex call instead.  Either way each result depends only on (every output's n, K,
 * SM count) and x's row: row invariance over M = 1..128 and determinism hold as for nvfp4_gemv,
 * and the result of an output alone (count 1) is bitwise that of nvfp4_gemv_ex.  Output
 * buffers must not overlap one another, x or the weights.
 * Errors: NVFP4_ERR_NULL (outputs NULL, or as nvfp4_gemv for an output), NVFP4_ERR_SHAPE
 * (count out of range, or as nvfp4_gemv), and those of nvfp4_gemv_ex, checked output by output
 * before anything is enqueued. */
int nvfp4_gemv_multi(const nvfp4_output_t* outputs, int count, const void* x, int64_t ldx,
                     int m, int64_t k, void* workspace, size_t workspace_bytes, uint32_t flags,
                     cudaStream_t stream);

/* Input prologues: the transform of x that the decode step runs just before a projection,
 * applied while the GEMV stages x instead of in a launch of its own.  The decode plan launches
 * them as residual_add_rms_norm / rms_norm (before the attention and FFN projections) and
 * sigmoid_gate_mul (before the attention output projection) ("Blueprint - circuit executor"
 * page for qwen3.8-27b-nvfp4 on GB10, table "Kernels the plan launches"; the page names them,
 * the formulas are the standard RMS normalisation with a gain and the sigmoid output gate of
 * gated attention).  The GEMV then runs on x', every weight of the call on the same x':
 *
 *   NVFP4_PROLOGUE_ADD_RMSNORM:   h[m][k]  = bf16_rn(x[m][k] + residual[m][k])
 *                                 x'[m][k] = bf16_rn(h[m][k] * inv(m) * gamma[k]),
 *                                 inv(m)   = 1 / sqrt(sum_k h[m][k]^2 / K + eps)
 *                                 and h is written to residual_out when that is not NULL.
 *   NVFP4_PROLOGUE_SIGMOID_GATE:  x'[m][k] = bf16_rn(x[m][k] / (1 + e^-gate[m][k]))
 *   NVFP4_PROLOGUE_GATED_RMSNORM: x is fp32 [M][ldx] for this kind (the GatedDeltaNet's
 *                                 output, "gated_rms_norm_f32_input" on the same page), and
 *                                 every group of G = `group` channels is normalised alone:
 *                                 x'[m][k] = bf16_rn(x[m][k] * inv(m, g) * gamma[k mod G]
 *                                                    * silu(gate[m][k])),
 *                                 inv(m, g) = 1 / sqrt(sum_{k in g} x[m][k]^2 / G + eps),
 *                                 silu(t) = t / (1 + e^-t).  G % 128 == 0, G <= 512,
 *                                 K % G == 0; NVFP4_FLAG_WIDE_TENSOR is ignored (8-row passes).
 *
 * in fp32 (h exactly rounded; the sum of squares in a fixed order).  gamma multiplies as given:
 * a checkpoint that stores (gamma - 1) passes 1 + its weights.  Row invariance over M = 1..128
 * and determinism hold as without a prologue, and h is bitwise the rounded sum.
 */
typedef enum {
    NVFP4_PROLOGUE_NONE = 0,
    NVFP4_PROLOGUE_ADD_RMSNORM = 1,
    NVFP4_PROLOGUE_SIGMOID_GATE = 2,
    NVFP4_PROLOGUE_GATED_RMSNORM = 3
} nvfp4_prologue_kind;

typedef struct {
    int32_t kind;            /* nvfp4_prologue_kind */
    float eps;               /* ADD_RMSNORM, GATED_RMSNORM: finite, >= 0 */
    const void* residual;    /* ADD_RMSNORM: bf16 [M][ld_residual] */
    int64_t ld_residual;
    const void* gamma;       /* ADD_RMSNORM: bf16 [K]; GATED_RMSNORM: bf16 [G] */
    void* residual_out;      /* ADD_RMSNORM: bf16 [M][ld_residual_out] receives h, or NULL */
    int64_t ld_residual_out;
    const void* gate;        /* SIGMOID_GATE, GATED_RMSNORM: bf16 [M][ld_gate] */
    int64_t ld_gate;
    int32_t group;           /* GATED_RMSNORM: channels per group, G (gamma is bf16 [G]) */
} nvfp4_prologue_t;

/* nvfp4_gemv_ex, nvfp4_gemv_dual_ex and nvfp4_gemv_multi with an input prologue.  `prologue`
 * is host memory read during the call only; NULL or kind NVFP4_PROLOGUE_NONE gives bitwise the
 * call without one.  The prologue runs as a grid of its own ahead of the GEMV on `stream` (one
 * CTA per row writes x' into the workspace, which must then hold nvfp4_workspace_bytes_wide(N,
 * K, M) bytes; with NVFP4_FLAG_PREFETCH_WEIGHTS the GEMV's weights stream in meanwhile), so
 * x' of a row is computed once and the GEMV's result is that of nvfp4_gemv on x'.  The
 * prologue's arrays are device memory: every row 16-byte aligned (base 16-byte aligned,
 * leading dimension >= K and a multiple of 8), like x.  residual_out may not
 * overlap x, residual, gamma or any y, and residual may not overlap y: NVFP4_ERR_ALIAS (the
 * prologue may read x and the residual again after writing h, and y is written after it; so
 * the residual is not updated in place).  With NVFP4_FLAG_WIDE_TENSOR the tier's x pass
 * applies the residual add + RMS norm and the sigmoid gate itself, and its rows are invariant
 * over 9..128 as without one.
 * Errors: those of the call without a prologue, and NVFP4_ERR_SHAPE (unknown kind, eps
 * negative or not finite, a leading dimension < K, a group size out of range or not dividing
 * K), NVFP4_ERR_NULL (a required array NULL when K > 0), NVFP4_ERR_ALIGN, NVFP4_ERR_ALIAS, all
 * checked before anything is enqueued. */
int nvfp4_gemv_pro(const nvfp4_prologue_t* prologue, const uint8_t* w, const uint8_t* s,
                   float global_scale, const void* x, int64_t ldx, void* y, int64_t ldy, int m,
                   int64_t n, int64_t k, void* workspace, size_t workspace_bytes, uint32_t flags,
                   cudaStream_t stream);
int nvfp4_gemv_dual_pro(const nvfp4_prologue_t* prologue, const uint8_t* w_gate,
                        const uint8_t* s_gate, float global_gate, const uint8_t* w_up,
                        const uint8_t* s_up, float global_up, const void* x, int64_t ldx,
                        void* y, int64_t ldy, int m, int64_t n, int64_t k, void* workspace,
                        size_t workspace_bytes, uint32_t flags, cudaStream_t stream);
int nvfp4_gemv_multi_pro(const nvfp4_prologue_t* prologue, const nvfp4_output_t* outputs,
                         int count, const void* x, int64_t ldx, int m, int64_t k,
                         void* workspace, size_t workspace_bytes, uint32_t flags,
                         cudaStream_t stream);

/* nvfp4_gemv for a caller that cannot provide a workspace.  The NVFP4 pages describe no such
 * call: it is a library convenience.  It serves callers that may not allocate device memory
 * and hold no buffer to lend: a plugin inside a host program that owns every device
 * allocation, or a C program whose device memory is all committed before its first GEMV
 * (cudaMalloc there would take memory outside that budget and synchronise the device).
 *
 * Arguments, layout, guarantees and results are those of nvfp4_gemv with flags 0; the
 * workspace is replaced by a scratch array compiled into this library (2,622,720 bytes of
 * device memory on each device that loads it: an error word, one hand-off word per CTA and two
 * pairs of fp32 partial tiles per CTA, for grids of up to 160 CTAs).  The call allocates
 * nothing.
 *
 * Set-up: every call (made with the intended device current) looks up the array's device
 * address in the current context with cudaGetSymbolAddress, a host-side lookup that allocates
 * nothing; the first call on a device may also load the library's module there, so make that
 * first call before any stream capture.  NVFP4_ERR_LAUNCH if the lookup fails.
 *
 * Sharing: every call on a device uses the same array and finds it as the previous call left
 * it.  Each call therefore first clears the error word and the hand-off words (a
 * cudaMemsetAsync of the first 1,280 bytes on `stream` on a 148-SM B200), then launches.  Calls that overlap in time -- on different
 * streams, or from different host threads -- race on the array and give wrong results:
 * issue them in one stream's order.  If a bounded wait inside the kernel gives up, the kernel
 * records it in the array's error word, which this call cannot report; callers that need
 * that check use nvfp4_gemv with nvfp4_workspace_error.
 *
 * Errors: NVFP4_ERR_WORKSPACE if the device has more than 160 SMs (the array is too small:
 * use nvfp4_gemv); otherwise those of nvfp4_gemv. */
int nvfp4_gemv_noalloc(const uint8_t* w, const uint8_t* s, float global_scale, const void* x,
                       int64_t ldx, void* y, int64_t ldy, int m, int64_t n, int64_t k,
                       cudaStream_t stream);

/* Chains: up to NVFP4_CHAIN_MAX_OPS GEMV operations in one persistent launch, run in order,
 * an operation optionally reading an earlier one's result as its x.  The decode plan runs its
 * projections as separate launches ("Blueprint - circuit executor" page, table "Kernels the
 * plan launches": w4a16_gemv_dual x64 feeding w4a16_gemv_sw, the MLP's gate_up and down); a
 * launch's fixed start and drain then cost more HBM time than a small projection streams.  In
 * a chain the weight stream continues across the boundaries: while one operation finishes,
 * the next one's weights already stream into shared memory (they do not depend on earlier
 * results).  An operation with x_from >= 0 waits on the device, per CTA, until every row group
 * of that earlier operation is written, then reads it.
 *
 * Every operation's result is bitwise that of the same call made alone (nvfp4_gemv_multi for
 * NVFP4_OP_SINGLE, nvfp4_gemv_dual for NVFP4_OP_DUAL, on the same x): each keeps its own work
 * split.  Row invariance over M = 1..128 and determinism therefore hold as for those calls.
 */
#define NVFP4_CHAIN_MAX_OPS 16
#define NVFP4_OP_SINGLE 0 /* 1..NVFP4_MAX_OUTPUTS weights sharing x (nvfp4_gemv_multi) */
#define NVFP4_OP_DUAL 1   /* silu(gate x) * (up x) (nvfp4_gemv_dual) */

typedef struct {
    int32_t kind;    /* NVFP4_OP_SINGLE or NVFP4_OP_DUAL */
    int32_t outputs; /* NVFP4_OP_SINGLE: 1..NVFP4_MAX_OUTPUTS; NVFP4_OP_DUAL: 1 */
    /* NVFP4_OP_SINGLE: the outputs, each N >= 1.  NVFP4_OP_DUAL: out[0] is the gate weight and
     * the result o (y, ldy, n), out[1] the up weight (its n must equal out[0].n; its y and ldy
     * are ignored). */
    nvfp4_output_t out[NVFP4_MAX_OUTPUTS];
    const void* x;   /* bf16 [M][ldx], used when x_from < 0 */
    int64_t ldx;
    int64_t k;       /* K of every weight of the operation: K % 256 == 0 */
    int32_t x_from;  /* -1: x as given.  j in [0, this operation's index): x is operation j's
                        result (j must have one output, with n == this K, y 16-byte aligned
                        and ldy % 8 == 0; x and ldx are then ignored) */
} nvfp4_chain_op_t;

/* Workspace bytes of nvfp4_gemv_chain for these operations and M (host only, besides the
 * device's SM count): a header and, per kernel operation, one hand-off word and two partial
 * tiles (per weight stream) per SM -- about 1.2 MB per single operation and 2.4 MB per dual on
 * a 148-SM B200.  Errors as nvfp4_gemv_chain's argument checks, and NVFP4_ERR_ARCH. */
int nvfp4_chain_workspace_bytes(const nvfp4_chain_op_t* ops, int count, int m, size_t* bytes);

/* Runs `count` (1..NVFP4_CHAIN_MAX_OPS) operations in order, M (1..128) rows each, one kernel
 * launch per 8-row pass.  ops is host memory read during the call only.  Per operation, the
 * rules of nvfp4_gemv_multi / nvfp4_gemv_dual hold, plus: K % 256 == 0 and every scale array
 * 16-byte aligned (the scale codes move by TMA).  An operation whose row groups exceed one
 * launch at its K (only for K above 9,728 with more than 10,496 rows) is cut into row chunks
 * as nvfp4_gemv cuts it; the chain may then hold at most NVFP4_CHAIN_MAX_OPS chunks in all.
 * Outputs may not overlap one another, any x or any weight: operations run concurrently on
 * different SMs, ordered only through x_from.
 *   workspace: 16-byte aligned, nvfp4_chain_workspace_bytes(ops, count, m) bytes, zero-filled
 *     before first use; reset by every completed launch, as for nvfp4_gemv.
 *   flags: 0 or NVFP4_FLAG_PREFETCH_WEIGHTS (the chain's first weights stream in while the
 *     kernel before it finishes).
 * A chain with x_from links is launched cooperatively (all CTAs resident at once), so its
 * waits always end; each wait still gives up after 1 s and then sets the workspace's error word
 * to 4 (results invalid; nvfp4_workspace_error reads it).
 * Errors: NVFP4_ERR_NULL, NVFP4_ERR_SHAPE (count, kind, outputs, K, x_from out of range or its
 * source not one output of N == K, too many chunks, unknown flags), NVFP4_ERR_ROWS,
 * NVFP4_ERR_ALIGN, NVFP4_ERR_WORKSPACE, NVFP4_ERR_ARCH, NVFP4_ERR_LAUNCH; all checked before
 * anything is enqueued. */
int nvfp4_gemv_chain(const nvfp4_chain_op_t* ops, int count, int m, void* workspace,
                     size_t workspace_bytes, uint32_t flags, cudaStream_t stream);

/* Test form of nvfp4_gemv_chain, for the bounded waits: the first operation that a later one
 * reads never reports its completion, and the waits give up after wait_limit_ns (1 .. 1e9).
 * The launch then ends normally with error word 4 in the workspace and that reader's outputs
 * invalid; the device stays usable.  No other use. */
int nvfp4_gemv_chain_unsignalled(const nvfp4_chain_op_t* ops, int count, int m, void* workspace,
                                 size_t workspace_bytes, int64_t wait_limit_ns,
                                 cudaStream_t stream);

/* Test form of nvfp4_gemv_chain, for the hand-off of cut row groups: the CTA holding a group's
 * first unit waits at most owner_wait_ns (0 .. 50000) for the later CTAs' partial sums before it
 * publishes its own and leaves the group to the last of them (50000 is nvfp4_gemv_chain's
 * limit).  With 0 nearly every cut group takes that path.  Results are bitwise those of
 * nvfp4_gemv_chain.  No other use. */
int nvfp4_gemv_chain_owner_wait(const nvfp4_chain_op_t* ops, int count, int m, void* workspace,
                                size_t workspace_bytes, int64_t owner_wait_ns,
                                cudaStream_t stream);

/* Workspace bytes of an nvfp4_gemv_ex / _pro, nvfp4_gemv_dual_ex / _pro or nvfp4_gemv_multi /
 * _pro (the largest of its outputs' sizes) call of M rows with
 * NVFP4_FLAG_WIDE_TENSOR or an input prologue: the nvfp4_workspace_bytes layout followed by the
 * larger of the tier's scratch (fp32 partial sums of its split of K, an f16 copy of x with the
 * rows' scales, and the dual's two fp32 results; the size depends on N, K, M and the SM count)
 * and the prologue's x' (M x K bf16).  Zero-filled before first use, like any workspace.
 * NVFP4_ERR_NULL, NVFP4_ERR_SHAPE (as nvfp4_gemv), NVFP4_ERR_ROWS, NVFP4_ERR_ARCH. */
int nvfp4_workspace_bytes_wide(int64_t n, int64_t k, int m, size_t* bytes);

/* The workspace's error word after the work enqueued so far has run (synchronises the
 * stream): 0 if no kernel hit a bounded wait's limit, else a nonzero code -- 2 or 3: a wait on
 * the shared-memory ring (a weight copy that never landed), 4: a chain's dependency wait --
 * and the results of the call that set it are invalid (zero-fill the workspace before reuse).
 * Returns NVFP4_OK and writes *error, or an nvfp4_status error. */
int nvfp4_workspace_error(const void* workspace, size_t workspace_bytes, cudaStream_t stream,
                          int32_t* error);

/* Human-readable name of a status code (static string). */
const char* nvfp4_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* NVFP4_H */
