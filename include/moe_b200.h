/*
 * moe_b200.h -- C ABI of libmoe_b200.so: the quantized routed-expert MoE
 * layer call on one NVIDIA B200 (sm_100a).
 *
 * One call computes, for M tokens of hidden size H, E experts, top-k routing
 * and per-expert intermediate size I:
 *   route    s = sigmoid(logits); top-k of s + bias (ties -> lower expert ID);
 *            w_j = s_j / sum_j s_j * routed_scale
 *   align    the M*k (token, slot) pairs sorted stably by expert
 *   quant    x -> MXFP4 (E2M1 + E8M0 per 32) for MXFP4 weights,
 *            x -> E4M3 + power-of-two fp32 scale per 128 for block-FP8 weights
 *   GEMM1    g = x_q . w13[e]^T, rows [0, I) gate and [I, 2I) up
 *   SwiGLU   mid = silu(gate) * up, quantized once to E4M3 with one
 *            power-of-two fp32 scale per 128 values of one pair
 *   GEMM2    y = mid_q . w2[e]^T
 *   combine  out[t] = bf16( sum_j w_j * y[t, j] ), j ascending, deterministic
 *
 * Passages defining the operation (page title, section):
 *   - "glm53: FP8 mid hand-off, ..." (MarloweAI/sgl-amd-mono-upstream PR 21),
 *     Modifications table row 1 and the commit "Quantize each mid block to
 *     FP8 once": mid is quantized to FP8 once per block, with a scale, and
 *     every down task reads the FP8 bytes; commit "per-row up/gate jobs at 4
 *     rows": top-8 rounds, a tied round broken by expert ID.
 *   - "glm53_flash: score a verify request's index tiles once" (sgl-amd-mono
 *     PR 100), commit message: above 8 rows the MoE runs expert-major, each
 *     expert's weights read once for all rows that pick it.
 *   - "IQ2R: load GLM-5.3 packed MoE checkpoints with TP slicing" (ROCm/ATOM
 *     PR 2335), benchmark notes: the MXFP4 arm is A4W4 (activations FP4 too);
 *     the MoE method runs after the usual expert selection, SiLU activation.
 *   - "[HIP] IQ2R: GLM-5.3 packed MoE path for TP4/TP8 on gfx950"
 *     (ROCm/aiter PR 5728), Technical Details: 256 routed experts, hidden
 *     6144, per-rank intermediate 512 (TP4) / 256 (TP8); launchers run on the
 *     tensors' device (device guard).
 *   Weight formats: OCP Microscaling Formats v1.0 (MXFP4) and OCP 8-bit
 *   floating point (E4M3) with one fp32 scale per 128x128 block.
 *
 * Conventions for every entry point:
 *   - All tensor pointers are DEVICE pointers on the device that owns
 *     `stream` (a cudaStream_t passed as void*; NULL = legacy default stream).
 *     The library switches to that device for the call and restores the
 *     caller's current device before returning.  While `stream` is being
 *     captured into a CUDA graph the stream cannot be asked for its device:
 *     the caller's current device is used and pointers are not re-checked.
 *   - Calls are stream-ordered and asynchronous: no entry point except
 *     moe_get_status synchronizes.  Buffers must stay alive until the stream
 *     has passed the call.
 *   - The caller owns every buffer, including the workspace.  No entry point
 *     allocates device memory.  The library keeps no per-call global state; a
 *     workspace serves one stream at a time.
 *   - Row-major, K (the contracted dimension) contiguous.  Two E2M1 values per
 *     byte: element 2i in bits 3:0, element 2i+1 in bits 7:4.  bf16 tensors
 *     are passed as raw 16-bit patterns.  Base pointers 256-byte aligned.
 *   - Argument errors are detected on the host before any launch and return
 *     a negative moe_status_t; nothing is launched then.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = -1,     /* null pointer, bad shape, misaligned buffer   */
  MOE_ERR_UNSUPPORTED = -2,     /* shape outside the supported limits           */
  MOE_ERR_WORKSPACE = -3,       /* workspace smaller than moe_workspace_size    */
  MOE_ERR_DEVICE_MISMATCH = -4, /* a pointer lives on another device            */
  MOE_ERR_CUDA = -5,            /* a CUDA runtime/driver call failed            */
  MOE_ERR_DEVICE_TIMEOUT = -6   /* a bounded device-side wait ran out           */
} moe_status_t;

typedef enum { MOE_W_MXFP4 = 1, MOE_W_FP8_BLOCK128 = 2 } moe_wfmt_t;

/* Shape limits: M >= 1; H % 256 == 0 (MXFP4) or H % 128 == 0 (FP8);
 * I % 128 == 0; 1 <= topk <= min(E, 16); E <= 512; M * topk <= 2^20.    */
typedef struct {
  int32_t M, H, I, E, topk;
  float routed_scale;
  int32_t wfmt;               /* moe_wfmt_t */
} moe_shape_t;

/* Byte offsets of the debug taps inside a workspace.  After moe_forward the
 * workspace holds, at these offsets (P = M*topk pairs, "sorted" = the
 * expert-major order of moe_forward's align step):
 *   topk_ids     int32 [M][topk]        expert of each (token, slot)
 *   topk_w       fp32  [M][topk]        routing weight of each (token, slot)
 *   counts       int32 [E]              pairs per expert
 *   offsets      int32 [E+1]            exclusive prefix of counts
 *   sorted_pairs int32 [P]              pair id p = t*topk + j at each sorted slot
 *   inv          int32 [P]              sorted slot of each pair
 *   midq         uint8 [P][I]           E4M3 mid codes, rows in sorted order
 *   midqs        fp32  [P][I/128]       power-of-two mid scales, sorted order
 *   status       int32 [4]              [0] device status word (see moe_get_status),
 *                                       [2] first timed-out wait: 0x8 | kernel<<24 |
 *                                       site<<20 | stage<<12 | CTA (diagnosis) */
typedef struct {
  uint64_t status, topk_ids, topk_w, counts, offsets, sorted_pairs, inv;
  uint64_t midq, midqs, total_bytes;
} moe_ws_layout_t;

/* Workspace bytes moe_forward needs for `shape` (host only, pure).
 * Returns MOE_OK, MOE_ERR_INVALID_ARG or MOE_ERR_UNSUPPORTED.              */
MOE_API int moe_workspace_size(const moe_shape_t* shape, size_t* bytes);

/* Offsets of the debug taps (host only, pure).                             */
MOE_API int moe_workspace_layout(const moe_shape_t* shape, moe_ws_layout_t* layout);

/* Zero-fill a workspace.  A workspace must be zero-filled once before its
 * first moe_forward; the library leaves its counters at zero after every
 * call, so later calls of the same shape need no re-initialization.  The
 * decode path tags its flags with a per-workspace call count, so a workspace
 * that moves to another shape (another layout) must be zero-filled again.  */
MOE_API int moe_workspace_init(void* workspace, size_t ws_bytes, void* stream);

/* Routing only: sigmoid + bias top-k selection and normalized weights.
 *   logits  fp32 [M][E]; bias fp32 [E] or NULL (zero bias)
 *   topk_ids int32 [M][topk] out, slot 0 the best; topk_w fp32 [M][topk] out
 * The sigmoid is computed with a specified fp32 operation sequence (Cody-
 * Waite exp, degree-7 polynomial) so the selection is reproducible bit for
 * bit.  Source: "glm53: FP8 mid hand-off", commit "per-row up/gate jobs".  */
MOE_API int moe_route(const moe_shape_t* shape, const float* logits, const float* bias,
              int32_t* topk_ids, float* topk_w, void* stream);

/* The whole MoE call.
 *   x          bf16 [M][H]
 *   logits     fp32 [M][E];  bias fp32 [E] or NULL
 *   MXFP4:  w13 uint8 [E][2I][H/2],  w13_scales: E8M0 [E][2I][H/32] packed
 *           w2  uint8 [E][H][I/2],   w2_scales:  E8M0 [E][H][I/32]  packed
 *           (packed = the layout moe_pack_mxfp4_scales writes, same size)
 *   FP8:    w13 uint8 (E4M3) [E][2I][H], w13_scales fp32 [E][2I/128][H/128]
 *           w2  uint8 (E4M3) [E][H][I],  w2_scales  fp32 [E][H/128][I/128]
 *   out        bf16 [M][H] (must not alias an input)
 *   workspace  >= moe_workspace_size bytes, zero-filled once (see above)
 * w13/w2 base pointers must be 32-byte aligned, all others 16-byte aligned.
 * Device-side waits are bounded; if one runs out the kernel records it in the
 * workspace status word and returns early (moe_get_status reports it).     */
MOE_API int moe_forward(const moe_shape_t* shape, const void* x, const float* logits,
                const float* bias, const void* w13, const void* w13_scales,
                const void* w2, const void* w2_scales, void* out,
                void* workspace, size_t ws_bytes, void* stream);

/* The MoE call after expert selection made by the caller (the pages' op runs
 * after "the usual expert selection"): the same call as moe_forward with the
 * routing step replaced by the caller's choice.
 *   topk_ids  int32 [M][topk], expert IDs in [0, E); a token may name an
 *             expert more than once, and each occurrence counts
 *   topk_w    fp32  [M][topk], the weights the combine applies as given
 * Everything else (x, weights, out, workspace) as moe_forward; 16-byte
 * aligned.  The IDs are read on the device: one outside [0, E) makes the
 * call record ST_BAD_INPUT in the workspace status word and use expert 0
 * with weight 0 for that slot, so it still ends normally; out is then
 * unspecified and moe_get_status returns MOE_ERR_INVALID_ARG.  The debug
 * taps hold the (replaced) selection.  Source: "IQ2R: load GLM-5.3 packed
 * MoE checkpoints" (the interface: an op after expert selection, with a
 * caller-provided workspace).                                             */
MOE_API int moe_forward_routed(const moe_shape_t* shape, const void* x, const int32_t* topk_ids,
                               const float* topk_w, const void* w13, const void* w13_scales,
                               const void* w2, const void* w2_scales, void* out,
                               void* workspace, size_t ws_bytes, void* stream);

/* One tensor-parallel rank's share of the call: the same call as moe_forward
 * on the rank's slice of every expert's intermediate dimension, leaving the
 * rank's fp32 sum instead of bf16 out.
 *   shape->I   the slice width I/T (a multiple of 128: the mid blocks of 128
 *              and the weight blocks stay whole)
 *   w13        the slice's gate rows followed by its up rows, [E][2 I/T][...]
 *   w2         the slice's columns, [E][H][I/T ...] (packed scales alike)
 *   out_partial fp32 [M][H]; 16-byte aligned
 * Every rank routes the same logits to the same selection (routing does not
 * depend on I), so the sum over the T ranks of out_partial, rounded to bf16
 * (moe_round_bf16), is the unsplit call's output up to fp32 summation order.
 * That sum is the caller's collective (an all-reduce over the ranks).  Other
 * arguments as moe_forward.  Source: "glm53: FP8 mid hand-off" (Accuracy
 * Tests: a rank's partial sums meet its peers'); "[HIP] IQ2R: GLM-5.3 packed
 * MoE path for TP4/TP8" (per-rank intermediate 512 at TP4, 256 at TP8).   */
MOE_API int moe_forward_partial(const moe_shape_t* shape, const void* x, const float* logits,
                                const float* bias, const void* w13, const void* w13_scales,
                                const void* w2, const void* w2_scales, float* out_partial,
                                void* workspace, size_t ws_bytes, void* stream);

/* Tensor-core throughput of this GPU for one MMA kind, measured: every SM
 * issues `iters` blocks of four M = 128, N = 128 tcgen05 MMAs back to back on
 * operands resident in shared memory (values 1.0, block scales 2^0), timed on
 * the device up to the completion of the last one.  The figure is the
 * denominator of the call's tensor fraction (the pages time their kernels
 * against counters checked on a workload of known size: "IQ2R: load GLM-5.3
 * packed MoE checkpoints with TP slicing", single-GPU MoE results).
 *   kind          MOE_PROBE_FP8  (kind::f8f6f4, E4M3 x E4M3: the block-FP8
 *                                GEMMs and MXFP4 GEMM2's 8-bit operand rate)
 *                 MOE_PROBE_FP4  (kind::mxf4, E2M1 x E2M1 with E8M0 per 32:
 *                                MXFP4 GEMM1)
 *                 MOE_PROBE_BF16 (kind::f16 with bf16 operands, for comparison
 *                                with a bf16 GEMM peak)
 *   iters         1 .. 100000 blocks per SM (2000 take ~0.3 ms at FP8)
 *   tflops        out: 2 x MACs of all SMs over the slowest SM's time, TFLOP/s
 *   mac_per_clk   out: MACs per SM clock of the median SM
 * A shorter warm-up run precedes the timed one.  Synchronizes `stream` (not
 * capturable in a CUDA graph); allocates nothing (a small static device
 * array holds the per-SM timings, so probes overlapping on one device race
 * on it: run one at a time per device).  Returns MOE_ERR_INVALID_ARG for a bad kind
 * or count, a null output or a capturing stream, MOE_ERR_CUDA on a CUDA
 * error, MOE_ERR_DEVICE_TIMEOUT if the last MMA's completion was not seen.   */
enum { MOE_PROBE_FP8 = 0, MOE_PROBE_FP4 = 1, MOE_PROBE_BF16 = 2 };
MOE_API int moe_probe_tensor_peak(int kind, int iters, double* tflops, double* mac_per_clk, void* stream);

/* bf16 (round to nearest even) of n fp32 values: out[i] = bf16(in[i]), for
 * the all-reduced partials of moe_forward_partial.  n % 8 == 0; both pointers
 * 16-byte aligned device memory on the stream's device.                     */
MOE_API int moe_round_bf16(const float* in, void* out, int64_t n, void* stream);

/* moe_forward that also records five CUDA events (cudaEvent_t as void*) on
 * `stream`: events[0] before the route kernel, events[1..4] after the route
 * and sort kernels, GEMM1, GEMM2 and combine -- per-step device times for
 * profiling.
 * The events separate the launches, so the kernels do not overlap their
 * prologues with the previous kernel's tail as they do in moe_forward.
 * Under stream capture the events become external event-record nodes, so a
 * replayed graph still timestamps them.  When the call runs as one kernel
 * (decode-sized MXFP4 batches), events[1..4] all follow that kernel.       */
MOE_API int moe_forward_timed(const moe_shape_t* shape, const void* x, const float* logits,
                              const float* bias, const void* w13, const void* w13_scales,
                              const void* w2, const void* w2_scales, void* out,
                              void* workspace, size_t ws_bytes, void* stream,
                              void* const* events);

/* Number of kernels one moe_forward of `shape` launches on `device`: 1 when
 * the call runs as the single decode-sized kernel (MXFP4 weights, M <= 16,
 * M * topk <= 64, I <= 1024, H <= 8192, and the device can hold its
 * clusters, at least one per two 128-row tiles of H), else 6 (route +
 * quantize + sort counts, sort scatter, operand-scale packing, GEMM1, GEMM2,
 * combine).  Host
 * query only: nothing is launched.  Returns MOE_ERR_INVALID_ARG for a null
 * pointer or a device index out of range, the make-plan error for a shape the
 * library does not support.                                                 */
MOE_API int moe_launches_per_call(const moe_shape_t* shape, int device, int* launches);

/* Synchronize `stream`, read the workspace status word into *device_status
 * and clear it.  Returns MOE_OK when it was zero, MOE_ERR_INVALID_ARG when a
 * caller-routed expert ID was out of range (moe_forward_routed),
 * MOE_ERR_DEVICE_TIMEOUT when a bounded wait ran out, MOE_ERR_CUDA on a CUDA
 * error.
 * Device-side waits (the single-launch path's flags between its CTAs) give up
 * after MOE_WAIT_TIMEOUT_MS milliseconds (environment, read once per
 * process; default 2000); the kernel then records the first timed-out wait in
 * status word [2] and returns early instead of trapping.  Test knob:
 * MOE_TEST_WITHHOLD_FLAG=n (read once per process) makes the first n
 * single-launch calls leave one mid flag unpublished, so that those waits run
 * out and the call reports MOE_ERR_DEVICE_TIMEOUT; the next call is normal.  */
MOE_API int moe_get_status(void* workspace, void* stream, int32_t* device_status);

/* Size of the scratch array behind moe_forward_static (8 MiB).            */
#define MOE_STATIC_SCRATCH_BYTES (8u << 20)

/* moe_get_status for the static scratch of moe_forward_static on the device
 * that owns `stream`: synchronizes the stream, returns (and clears) the status
 * word the last moe_forward_static call on that device left, with the same
 * return codes as moe_get_status.  Each moe_forward_static call clears the
 * status word when it starts, so query it after the call and before the next
 * one.  Its first use on a device looks up the static scratch like the first
 * moe_forward_static call (see below), so it can also serve as that set-up.  */
MOE_API int moe_get_status_static(void* stream, int32_t* device_status);

/* moe_forward for callers that cannot allocate device memory: code running
 * where cudaMalloc is not an option (inside a custom allocator or a memory-
 * pool callback, in a process whose device memory is fully reserved by
 * another runtime, or in a plugin that is handed only input and output
 * buffers).  It allocates nothing: its scratch is one fixed, zero-initialized
 * array of MOE_STATIC_SCRATCH_BYTES that the library holds on every device
 * that loads it until the process exits.  The caller still passes inputs and
 * outputs, with the same meaning and layout as moe_forward.
 *   - The first call on a device (or moe_get_status_static) looks up the
 *     array's device address with that device current; make that first call
 *     before any stream capture.  The CUDA runtime commits the array's device
 *     memory when it loads the library's module that holds it: with lazy
 *     module loading (the CUDA 12 default) that is this first look-up, so a
 *     caller that will later run without free device memory makes it at
 *     start-up, while memory is still available (moe_get_status_static on an
 *     idle stream does it without a launch).
 *   - Shapes whose scratch exceeds MOE_STATIC_SCRATCH_BYTES (moe_workspace_
 *     size) are rejected with MOE_ERR_WORKSPACE before any launch; decode-
 *     sized calls (a few to a few dozen tokens) fit.
 *   - Every call on a device shares the array and leaves its contents behind;
 *     each call clears what must start at zero.  Calls whose executions
 *     overlap on the GPU (different streams without ordering) race on it.
 *   - Device-side timeouts are reported by moe_get_status_static; the debug
 *     taps of moe_workspace_layout do not apply.
 * The pages' system has no counterpart of this entry point.               */
MOE_API int moe_forward_static(const moe_shape_t* shape, const void* x, const float* logits,
                               const float* bias, const void* w13, const void* w13_scales,
                               const void* w2, const void* w2_scales, void* out, void* stream);

/* Text describing the last failed call on the calling thread (the CUDA call
 * and its error string, or the rejected argument); "" if none failed yet.
 * The pointer stays valid until the thread's next library call.           */
MOE_API const char* moe_last_error(void);

/* Offline weight preparation (not part of the timed call).
 * MXFP4 of `rows` rows of K fp32 values (K % 32 == 0), OCP MX rule: scale
 * 2^(floor(log2 amax) - 2) as E8M0, elements E2M1 round-to-nearest-even,
 * saturating.  q: rows*K/2 bytes, scales: rows*K/32 bytes.                 */
MOE_API int moe_quantize_mxfp4(const float* w, int64_t rows, int32_t K,
                       uint8_t* q, uint8_t* scales, void* stream);

/* Rearranges the E8M0 scales of `batch` MXFP4 matrices [rows][K] from the
 * row-major layout moe_quantize_mxfp4 writes ([batch][rows][K/32]) into the
 * layout moe_forward reads, which the tensor cores' scale-factor copy takes
 * as is: per matrix, 128-row tiles; per tile, one 512-byte block for each 128
 * columns (4 scales per row); in a block, row r of the tile at byte
 * 16 * (r % 32) + 4 * (r / 32), its 4 scales in column order.  Blocks are
 * ordered [batch][rows/128][K/128], so a tile's blocks along K are
 * contiguous.  rows % 128 == 0, K % 128 == 0; scales 4-byte aligned, packed
 * 16-byte aligned, the two must not overlap.  Same byte count as the input.
 * The pages' MXFP4 format fixes only the values (one E8M0 per 32 elements,
 * OCP MX v1.0); this byte order is the library's.                         */
MOE_API int moe_pack_mxfp4_scales(const uint8_t* scales, int64_t batch, int32_t rows, int32_t K,
                                  uint8_t* packed, void* stream);

/* 128x128 block FP8 of `batch` matrices [rows][K] (rows, K % 128 == 0):
 * scale = amax/448 in fp32 (1 for an all-zero block), q = E4M3(w / scale)
 * round-to-nearest-even, saturating.  scales: [batch][rows/128][K/128].    */
MOE_API int moe_quantize_fp8_block128(const float* w, int64_t batch, int32_t rows,
                              int32_t K, uint8_t* q, float* scales, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* MOE_B200_H */
