/*
 * nvfp4.h -- C ABI of the B200 (sm_100a) NVFP4 W4A4 linear-layer library
 * (libnvfp4.so).
 *
 * The method: every linear layer of a hybrid LLM runs with 4-bit weights and
 * 4-bit activations in NVFP4, i.e. E2M1 codes where each group of 16
 * consecutive codes shares one E4M3 scale ("NVFP4 W4A4 quantization compresses 27B hybrid models",
 * thevalue.engineering, section "Challenging the Recurrence Fragility
 * Assumption"; "Why Gated DeltaNet Survives 4-Bit Quantization", kipquest.com,
 * "The abstract" and "The deep dive").  Checkpoints are calibrated per module,
 * each module carrying its own FP32 global scale; serving kernels fuse modules
 * that share an input (q/k/v/z/b/a, gate/up) into one GEMM, and the paper
 * repairs the global-scale mismatch this causes (same page, "The abstract",
 * "The deep dive").  This library applies each module's own global scale to
 * its column segment in the GEMM epilogue.
 *
 * Conventions shared by every entry point:
 *  - Pointers named X, W, codes, sf, g_*, out, ws are DEVICE pointers owned by
 *    the caller; the library never allocates or frees memory.  Pointers to
 *    nvfp4_segment arrays are HOST pointers, read before the call returns.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *    stream).  All work is asynchronous on that stream; nothing synchronizes
 *    except nvfp4_get_status().
 *  - Return value: an nvfp4_status.  Argument errors are detected on the host
 *    before anything is launched.  A failed launch returns NVFP4_ERR_CUDA.
 *    Errors found on the device (a bounded wait that ran out, non-finite
 *    input) are latched in a per-device status word read by
 *    nvfp4_get_status().  No kernel ever traps.
 *  - bf16 matrices are row-major; `ld*` arguments are leading dimensions in
 *    elements.  Base pointers must be 16-byte aligned and leading dimensions
 *    multiples of 8 elements (NVFP4_ERR_MISALIGNED otherwise).
 *  - Weights use the nn.Linear layout W[N, K]; a linear computes
 *    out[M, N] = X[M, K] * W^T.
 *  - Kernels are launched with programmatic stream serialization: each one
 *    waits (griddepcontrol.wait) for the work before it on the stream and
 *    then lets the next kernel start its set-up early.  Stream order is kept
 *    for every ordinary launch; a caller's own kernel launched after ours
 *    with cudaLaunchAttributeProgrammaticStreamSerialization must call
 *    cudaGridDependencySynchronize() before reading our outputs, as with any
 *    such launch.  Calls can be captured in CUDA graphs.
 *
 * NVFP4 storage produced and consumed here:
 *  - codes: [rows, K/2] bytes, row-major; byte i of a row holds element 2i in
 *    its low nibble and element 2i+1 in its high nibble (E2M1: sign bit 3,
 *    exponent bits 2..1, mantissa bit 0).
 *  - sf: E4M3 block scales in the 128x4 tile layout the block-scaled MMA
 *    reads: the logical [rows, K/16] scale matrix is padded to a multiple of
 *    128 rows and 4 block-columns (padding bytes are written as 0) and cut
 *    into 512-byte tiles; tile (rt, ct) lives at byte (rt*ceil(K/64) + ct)*512
 *    and, inside it, row r / block-column c sits at
 *    (r%32)*16 + ((r%128)/32)*4 + c%4.  Size: nvfp4_sf_bytes(rows, K).
 *  - global scale g (fp32, device): the decode multiplier, value ~= code *
 *    scale * g.  Dynamic scales are g = amax/(6*448) over the tensor (or the
 *    module segment), and g = 1 when amax == 0.
 *  - block scale s = E4M3_RNE_satfinite(fl32(fl32(bamax/6)/g)), element code =
 *    E2M1_RNE_satfinite(fl32(x / fl32(s*g))), +-0 when s == 0; ties go to the
 *    even code and negative values that round to zero keep their sign.
 */
#ifndef NVFP4_H_
#define NVFP4_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    NVFP4_OK = 0,
    NVFP4_ERR_INVALID_ARG = 1,       /* null pointer, negative size, bad segments, bad flags */
    NVFP4_ERR_UNSUPPORTED_SHAPE = 2, /* K not a multiple of 16 (quantize) / 64 (GEMM), too large */
    NVFP4_ERR_MISALIGNED = 3,        /* base pointer or leading dimension violates alignment */
    NVFP4_ERR_CUDA = 4,              /* a CUDA runtime call or launch failed */
    NVFP4_ERR_TIMEOUT = 5,           /* device: a bounded wait in a kernel ran out */
    NVFP4_ERR_NONFINITE = 6,         /* device: an input held Inf or NaN (outputs unspecified) */
    NVFP4_ERR_WORKSPACE = 7,         /* workspace missing or smaller than required */
    NVFP4_ERR_NO_DEVICE = 8          /* current device is not an sm_100 GPU */
} nvfp4_status;

/* A module's rows of a fused weight: half-open [n_begin, n_end).  Segment
 * tables must be sorted, contiguous and cover [0, N) exactly. */
typedef struct {
    int64_t n_begin;
    int64_t n_end;
} nvfp4_segment;

#define NVFP4_MAX_SEGMENTS 16

/* Flags. */
#define NVFP4_STATIC_SCALE 1u /* activation global scale is an input (calibrated), not computed */
#define NVFP4_OUT_FP32 2u     /* GEMM output is fp32 instead of bf16 */
#define NVFP4_DEBUG_INJECT_STALL (1u << 30) /* nvfp4_gemm_prequant only: the kernel's loads are
                               * skipped so its bounded waits run out (20 ms) and it
                               * unwinds, latching NVFP4_ERR_TIMEOUT; outputs are not
                               * written.  Exercises the failure path without a hang. */
#define NVFP4_SINGLE_CTA (1u << 29) /* GEMM entry points: use the one-CTA-per-tile kernel even
                               * where the CTA-pair kernel would run (M > 128).  Both
                               * compute the same block-scaled products; for tests and
                               * comparisons. */
#define NVFP4_AMAX_GIVEN 4u   /* nvfp4_quantize_act: the first word of ws already holds max|X|
                               * (bf16 magnitude bits, as nvfp4_gemm_prequant_swiglu leaves
                               * it); skip the amax pass */

/* Bytes of the swizzled scale-factor buffer for a [rows, K] matrix:
 * ceil(rows/128)*128 * ceil(K/64)*4.  Returns 0 for invalid sizes. */
size_t nvfp4_sf_bytes(int64_t rows, int64_t K);

/* Workspace bytes needed by nvfp4_quantize_act / nvfp4_quantize_weights /
 * nvfp4_swiglu_quantize (one amax word per segment, 256-byte aligned). */
size_t nvfp4_quant_workspace_bytes(int nseg);

/* Workspace bytes needed by nvfp4_linear / nvfp4_linear_fused for an [M, K]
 * input and N outputs: the quantized activation (codes and scale factors),
 * its amax and global scale and, for M <= 128 (decode-sized inputs), the
 * fp32 partial sums of the split-K GEMM (splits x M x N x 4 bytes, at most 8
 * splits; the split count depends on M, N and K only, so results do not
 * depend on the device).  nseg does not change the size and may be 0.  With
 * N = 0 the size covers the activation only, enough for every M > 128. */
size_t nvfp4_workspace_bytes(int64_t M, int64_t N, int64_t K, int nseg);

/* Offline weight quantization (post-training, per module).
 * W: bf16 [N, K] with leading dimension ldw; segs[nseg] (host) splits the N
 * rows into modules; each module m gets its own dynamic global scale
 * g_w[m] = amax_m/2688 (written to the device array g_w[nseg]).
 * Outputs: codes [N, K/2], sf (nvfp4_sf_bytes(N, K) bytes).  K % 16 == 0.
 * Passages: checkpoints whose modules were each calibrated with their own
 * scale (kipquest.com, "The abstract"); weights rounded after training rather than trained under
 * quantization (same page, "The deep dive"). */
int nvfp4_quantize_weights(const void *W, int64_t N, int64_t K, int64_t ldw,
                           const nvfp4_segment *segs, int nseg,
                           uint8_t *codes, uint8_t *sf, float *g_w,
                           void *ws, size_t ws_bytes, void *stream);

/* On-the-fly activation quantization (the A4 of W4A4).
 * X: bf16 [M, K], leading dimension ldx.  Outputs codes [M, K/2], sf
 * (nvfp4_sf_bytes(M, K) bytes).  Without NVFP4_STATIC_SCALE the global
 * scale is computed from max|X| and written to *g_a (device); with it, *g_a
 * is read as the calibrated scale.  K % 16 == 0.
 * Passage: NVFP4 W4A4 on all linear layers (kipquest.com, "The abstract"). */
int nvfp4_quantize_act(const void *X, int64_t M, int64_t K, int64_t ldx,
                       uint8_t *codes, uint8_t *sf, float *g_a, unsigned flags,
                       void *ws, size_t ws_bytes, void *stream);

/* Block-scaled FP4 GEMM on pre-quantized operands with the per-segment
 * global-scale epilogue:
 *   out[m, n] = round( acc[m, n] * fl32(g_a * g_w[seg(n)]) ),
 *   acc[m, n] = sum_k e2m1(a[m,k]) e4m3(sa[m,k/16]) e2m1(w[n,k]) e4m3(sw[n,k/16])
 * accumulated in fp32 on the tensor cores.  out is [M, N] row-major, bf16
 * (round to nearest even) or fp32 with NVFP4_OUT_FP32.  K % 64 == 0.
 * g_a: device, 1 float; g_w: device, nseg floats; segs: host.
 * Passage: serving separately calibrated modules through one fused GEMM,
 * and the global-scale repair (kipquest.com, "The abstract", "The deep dive"). */
int nvfp4_gemm_prequant(const uint8_t *a_codes, const uint8_t *a_sf, const float *g_a,
                        int64_t M, int64_t K,
                        const uint8_t *w_codes, const uint8_t *w_sf, int64_t N,
                        const nvfp4_segment *segs, const float *g_w, int nseg,
                        void *out, unsigned flags, void *stream);

/* nvfp4_gemm_prequant with a workspace: for M <= 128 the GEMM may divide K
 * among several CTAs (split-K, as nvfp4_linear_fused does; the fp32 partials
 * live in ws and are added in a fixed order).  ws: at least
 * nvfp4_gemm_workspace_bytes(M, N, K) bytes, 16-byte aligned (the size is 0
 * where no split is used; ws may then be NULL).  Use it where the activation
 * is already quantized at decode sizes, e.g. the down projection after
 * nvfp4_linear_swiglu. */
size_t nvfp4_gemm_workspace_bytes(int64_t M, int64_t N, int64_t K);
int nvfp4_gemm_prequant_ws(const uint8_t *a_codes, const uint8_t *a_sf, const float *g_a,
                           int64_t M, int64_t K,
                           const uint8_t *w_codes, const uint8_t *w_sf, int64_t N,
                           const nvfp4_segment *segs, const float *g_w, int nseg,
                           void *out, unsigned flags, void *ws, size_t ws_bytes, void *stream);

/* Fused-module linear: quantize X (as nvfp4_quantize_act, into the
 * workspace) then nvfp4_gemm_prequant against a fused weight whose rows are
 * split into nseg modules, each with its own global scale g_w[m].
 * X: bf16 [M, K] contiguous.  ws: nvfp4_workspace_bytes(M, N, K, nseg)
 * bytes.  With NVFP4_STATIC_SCALE the activation scale is read from the
 * first float of ws + 256 (see nvfp4_linear_act_scale_offset()).
 * Decode-sized inputs (M <= 128) may divide K among several CTAs (split-K):
 * each writes alpha * acc in fp32 to the workspace and a second kernel adds
 * the splits in a fixed order, so results are deterministic and the same on
 * every device, though their last bits can differ from nvfp4_gemm_prequant
 * (which never splits) on the same operands; both meet the same tolerance. */
int nvfp4_linear_fused(const void *X, int64_t M, int64_t K,
                       const uint8_t *w_codes, const uint8_t *w_sf, int64_t N,
                       const nvfp4_segment *segs, const float *g_w, int nseg,
                       void *out, unsigned flags, void *ws, size_t ws_bytes, void *stream);

/* Single-module linear: nvfp4_linear_fused with one segment [0, N). */
int nvfp4_linear(const void *X, int64_t M, int64_t K,
                 const uint8_t *w_codes, const uint8_t *w_sf, const float *g_w, int64_t N,
                 void *out, unsigned flags, void *ws, size_t ws_bytes, void *stream);

/* Byte offset inside a linear workspace of the activation global scale
 * (fp32): written by nvfp4_linear*, or read with NVFP4_STATIC_SCALE. */
size_t nvfp4_linear_act_scale_offset(void);

/* MLP intermediate of a gated MLP whose gate/up projections run as one fused
 * GEMM: h = bf16(silu(gate) * up) computed in fp32 from gate_up [M, 2F]
 * (leading dimension ld; gate = columns [0, F), up = [F, 2F)), written to
 * h [M, F] (contiguous), then quantized like nvfp4_quantize_act (codes
 * [M, F/2], sf, dynamic *g_h written).  F % 16 == 0.
 * Passage: gate/up fused into one GEMM (kipquest.com, "The abstract"); the
 * pages do not name the MLP activation, SiLU gating is the plain reading. */
int nvfp4_swiglu_quantize(const void *gate_up, int64_t M, int64_t F, int64_t ld,
                          void *h, uint8_t *codes, uint8_t *sf, float *g_h,
                          void *ws, size_t ws_bytes, void *stream);

/* Weights of a gated MLP for nvfp4_linear_swiglu: W is bf16 [2F, K] with the
 * gate projection in rows [0, F) and the up projection in rows [F, 2F); each
 * of the two modules gets its own dynamic global scale (g_w[0] gate, g_w[1]
 * up, device).  Codes and scales are stored with gate and up interleaved in
 * 128-row blocks -- gate rows [128b, 128b+128) at stored rows [256b,
 * 256b+128), up rows [128b, 128b+128) at [256b+128, 256b+256) -- so one
 * 256-row GEMM tile holds matching gate and up columns.  codes: [2F, K/2],
 * sf: nvfp4_sf_bytes(2F, K) bytes, ws: nvfp4_quant_workspace_bytes(2).
 * F % 128 == 0, K % 16 == 0.
 * Passage: gate/up are per-module-calibrated modules that serving kernels fuse
 * into one GEMM (kipquest.com, "The abstract", "The deep dive"). */
int nvfp4_quantize_weights_gated(const void *W, int64_t F, int64_t K, int64_t ldw,
                                 uint8_t *codes, uint8_t *sf, float *g_w,
                                 void *ws, size_t ws_bytes, void *stream);

/* The gated GEMM of nvfp4_linear_swiglu on already-quantized activations
 * (a_codes/a_sf/g_a as from nvfp4_quantize_act): writes h [M, F] bf16 and
 * leaves max|h| (bf16 magnitude bits) in the first word of ws (>= 256 bytes),
 * ready for nvfp4_quantize_act(h, ..., NVFP4_AMAX_GIVEN, ws, ...).
 * K % 64 == 0, F % 128 == 0. */
int nvfp4_gemm_prequant_swiglu(const uint8_t *a_codes, const uint8_t *a_sf, const float *g_a,
                               int64_t M, int64_t K, const uint8_t *w_codes, const uint8_t *w_sf,
                               int64_t F, const float *g_w, void *h, void *ws, size_t ws_bytes,
                               void *stream);

/* Gated-MLP up projection with the SwiGLU in the GEMM epilogue:
 *   h[m, j] = bf16_RNE( silu(gate) * up ),  silu(v) = v / (1 + exp(-v)),
 *   gate = fl32(acc_gate[m, j] * fl32(g_a * g_w[0])),
 *   up   = fl32(acc_up[m, j]   * fl32(g_a * g_w[1])),
 * with acc the fp32 block-scaled GEMM accumulators of X against the gate and
 * up rows of a weight from nvfp4_quantize_weights_gated (X is quantized on
 * the fly as in nvfp4_linear_fused; NVFP4_STATIC_SCALE reads its scale from the
 * workspace the same way).  Writes h [M, F] bf16 (contiguous), then quantizes
 * h for the next GEMM with its own dynamic scale: h_codes [M, F/2], h_sf
 * (nvfp4_sf_bytes(M, F) bytes), *g_h (device).  The epilogue folds max|h| in
 * as it writes h, so h is read once more, by the quantizer only.
 * ws: nvfp4_workspace_bytes(M, 2F, K, 2) bytes.  K % 64 == 0, F % 128 == 0.
 * Passage: the fused gate/up GEMM (kipquest.com, "The abstract"); the pages
 * do not name the MLP activation, SiLU gating is the plain reading. */
int nvfp4_linear_swiglu(const void *X, int64_t M, int64_t K,
                        const uint8_t *w_codes, const uint8_t *w_sf, int64_t F, const float *g_w,
                        void *h, uint8_t *h_codes, uint8_t *h_sf, float *g_h,
                        unsigned flags, void *ws, size_t ws_bytes, void *stream);

/* Synchronizes `stream`, then returns and clears the device status word of
 * the current device: NVFP4_OK, NVFP4_ERR_TIMEOUT or NVFP4_ERR_NONFINITE
 * (timeout wins when both are latched), or NVFP4_ERR_CUDA if the sync
 * failed. */
int nvfp4_get_status(void *stream);

/* Static, NUL-terminated description of a status code. */
const char *nvfp4_status_string(int status);

/* 1 if the current CUDA device is sm_100 (B200 class) and the library's
 * kernels can run on it, else 0. */
int nvfp4_device_supported(void);

/* Number of kernel launches (including memsets) the library has issued in
 * this process, for launch accounting. */
uint64_t nvfp4_launch_count(void);

/* Allocation-free variant of nvfp4_linear_fused (no counterpart in the
 * paper: this is a deployment convenience, not part of the method).
 *
 * Some callers cannot allocate device memory on the path that runs the
 * layer: a runtime or plugin host that owns every device allocation and
 * hands its operators no allocator, or a latency-critical serving loop in
 * which cudaMalloc's implicit device-wide synchronization is not allowed.
 * Such a caller cannot provide the scratch workspace that nvfp4_linear_fused
 * needs for the quantized activation.  This entry point keeps that scratch in
 * a fixed device array inside the library instead, and allocates nothing: it
 * calls no cudaMalloc / cudaFree and no allocating library routine.
 *
 * Arguments are those of nvfp4_linear_fused without the workspace; the
 * caller still passes X, the weight, the segment table and `out`.  Only the
 * dynamic activation scale is supported (NVFP4_STATIC_SCALE is rejected with
 * NVFP4_ERR_INVALID_ARG); NVFP4_OUT_FP32 is accepted.
 *
 * Limits: M*K <= NVFP4_NOALLOC_MAX_ELEMS and nvfp4_sf_bytes(M, K) <=
 * NVFP4_NOALLOC_MAX_SF_BYTES (about 2.5 MB of device memory, which every GPU
 * that loads the library keeps until the process exits).  Larger inputs are
 * rejected with NVFP4_ERR_WORKSPACE before anything is launched.
 *
 * The first call on a device looks up the array's device address (once per
 * device, with that device current); make that first call before any stream
 * capture begins.  All calls share the one array and it keeps the last
 * call's contents (no call reads what an earlier call left there): calls that can
 * overlap on the GPU -- on different streams without ordering, or from
 * several host threads -- race with each other and must be serialized by the
 * caller. */
#define NVFP4_NOALLOC_MAX_ELEMS (1ll << 22)
#define NVFP4_NOALLOC_MAX_SF_BYTES (1ll << 19)
int nvfp4_linear_fused_noalloc(const void *X, int64_t M, int64_t K,
                               const uint8_t *w_codes, const uint8_t *w_sf, int64_t N,
                               const nvfp4_segment *segs, const float *g_w, int nseg,
                               void *out, unsigned flags, void *stream);

/* ------------------------------------------------- FP8 KV-cache (E4M3)
 *
 * The attention KV cache in FP8 E4M3 with one calibrated FP32 scale per cache
 * tensor: the pages' recipe ships calibrated scales for the KV cache along
 * with the weights and reports them as costing nothing (freegardner.com, "Quantizing All
 * Layers Reveals Recurrent Memory Is Robust", section "The Calibrated Cache
 * That Ships for Free"; thevalue.engineering, "NVFP4 W4A4 quantization
 * compresses 27B hybrid models", section "Efficiency Gains and Serving
 * Optimization").  The pages give no formula; the reading used here:
 *   scale s = fl32(amax / 448) (1.0 when amax == 0), a decode multiplier,
 *   code    = E4M3 round-to-nearest-even, saturating at +-448, of fl32(x / s),
 *             the sign bit copying the sign of x.
 * X is bf16 [rows, cols] row-major with leading dimension ldx (elements);
 * cols % 8 == 0 (NVFP4_ERR_UNSUPPORTED_SHAPE otherwise), X 16-byte aligned
 * and ldx % 8 == 0 (NVFP4_ERR_MISALIGNED).  Any rows >= 0. */

/* Calibration: *scale (device fp32) = s for X.  ws: device workspace of at
 * least nvfp4_quant_workspace_bytes(1) bytes (its first word is overwritten).
 * Non-finite inputs latch NVFP4_ERR_NONFINITE (nvfp4_get_status). */
int nvfp4_fp8_kv_calibrate(const void *X, int64_t rows, int64_t cols, int64_t ldx, float *scale, void *ws,
                           size_t ws_bytes, void *stream);

/* Quantization with a calibrated scale: out[r, c] = code of X[r, c], out is
 * bytes [rows, cols] with leading dimension ldo (8-byte aligned base, ldo % 8
 * == 0).  scale: device fp32, read by the kernel; if it is not a positive
 * finite number nothing is written and NVFP4_ERR_NONFINITE is latched. */
int nvfp4_fp8_kv_quantize(const void *X, int64_t rows, int64_t cols, int64_t ldx, const float *scale, uint8_t *out,
                          int64_t ldo, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* NVFP4_H_ */
