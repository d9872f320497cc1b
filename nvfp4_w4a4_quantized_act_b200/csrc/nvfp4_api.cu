// nvfp4_api.cu -- the C ABI of libnvfp4.so: argument checks, workspace
// carving, TMA descriptor set-up and kernel launches for the NVFP4 W4A4
// linear layer.  Every entry point is declared and documented in
// include/nvfp4.h.
#include <algorithm>
#include <atomic>
#include <cstdint>
#include <cstring>
#include <mutex>

#include <cuda.h>
#include <cuda_runtime.h>

#include "nvfp4.h"
#include "gemm_kernel.cuh"
#include "gemm_pair_kernel.cuh"
#include "kv_cache_kernels.cuh"
#include "quantize_kernels.cuh"

namespace {

using nvfp4::kMaxSeg;

__device__ uint32_t g_status_word;  // per-device latched error bits

std::atomic<uint64_t> g_launches{0};

constexpr int kMaxDevices = 64;

struct DeviceState {
    bool init = false;
    bool supported = false;
    int sm_count = 0;
    uint32_t *status = nullptr;  // device address of g_status_word
    bool gemm_attr_set = false;
};

DeviceState g_dev[kMaxDevices];
std::mutex g_mu;

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;

// Looks up (once per device) the SM count, the status word address and
// whether the device is an sm_100 part.  Returns nullptr on failure.
DeviceState *device_state()
{
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
        return nullptr;
    DeviceState &d = g_dev[dev];
    if (d.init)
        return &d;
    std::lock_guard<std::mutex> lock(g_mu);
    if (d.init)
        return &d;
    cudaDeviceProp prop;
    if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess)
        return nullptr;
    d.supported = (prop.major == 10 && prop.minor == 0);
    d.sm_count = prop.multiProcessorCount;
    if (d.supported) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_status_word) != cudaSuccess)
            return nullptr;
        d.status = static_cast<uint32_t *>(p);
        if (cudaFuncSetAttribute(nvfp4::gemm::gemm_nvf4_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 nvfp4::gemm::SMEM_BYTES) != cudaSuccess ||
            cudaFuncSetAttribute(nvfp4::gemm::gemm_nvf4_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 nvfp4::gemm::SMEM_BYTES) != cudaSuccess ||
            cudaFuncSetAttribute(nvfp4::gemm::pair::gemm_nvf4_pair_kernel<false>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, nvfp4::gemm::pair::SMEM_BYTES) != cudaSuccess ||
            cudaFuncSetAttribute(nvfp4::gemm::pair::gemm_nvf4_pair_kernel<true>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, nvfp4::gemm::pair::SMEM_BYTES) != cudaSuccess)
            return nullptr;
        d.gemm_attr_set = true;
        if (g_encode == nullptr) {
            void *fn = nullptr;
            cudaDriverEntryPointQueryResult q;
            if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
                q != cudaDriverEntryPointSuccess || fn == nullptr)
                return nullptr;
            g_encode = reinterpret_cast<EncodeTiledFn>(fn);
        }
    }
    d.init = true;
    return &d;
}

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline int64_t round_up(int64_t a, int64_t b) { return (a + b - 1) / b * b; }
inline int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }

int64_t sf_bytes_i(int64_t rows, int64_t K) { return round_up(rows, 128) * cdiv(K / 16, 4) * 4; }

int check_segments(const nvfp4_segment *segs, int nseg, int64_t N, nvfp4::SegRows *out)
{
    if (segs == nullptr || nseg < 1 || nseg > kMaxSeg)
        return NVFP4_ERR_INVALID_ARG;
    int64_t expect = 0;
    out->nseg = nseg;
    for (int i = 0; i < nseg; ++i) {
        if (segs[i].n_begin != expect || segs[i].n_end < segs[i].n_begin)
            return NVFP4_ERR_INVALID_ARG;
        expect = segs[i].n_end;
        out->end[i] = segs[i].n_end;
    }
    for (int i = nseg; i < kMaxSeg; ++i)
        out->end[i] = N;
    return expect == N ? NVFP4_OK : NVFP4_ERR_INVALID_ARG;
}

thread_local bool t_launch_failed = false;

// Launches a kernel with programmatic stream serialization: the kernel may
// be scheduled while the previous kernel on the stream is still running and
// waits for it (griddepcontrol.wait) before touching global memory.  Every
// kernel of this library does that wait first, so stream order holds.
template <typename... KArgs, typename... Args>
void launch(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream, Args... args)
{
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, kernel, args...) != cudaSuccess)
        t_launch_failed = true;
}

int launch_ok()
{
    const bool failed = t_launch_failed;
    t_launch_failed = false;
    return (cudaGetLastError() == cudaSuccess && !failed) ? NVFP4_OK : NVFP4_ERR_CUDA;
}

// Clears `n` amax words on the stream (a kernel, so that the launches around
// it keep their programmatic dependencies).
int zero_words(uint32_t *words, int n, cudaStream_t stream)
{
    launch(nvfp4::zero_words_kernel, dim3(1), dim3(32), 0, stream, words, static_cast<int32_t>(n));
    g_launches++;
    return launch_ok();
}

// Rows of the amax pass are cut into ranges of 128 16-byte chunks (one
// four-load sweep of a warp) while rows are too few to give every SM work.
int64_t amax_slices(int64_t rows, int64_t cols)
{
    if (rows >= 1024)
        return 1;
    return std::max<int64_t>(1, cdiv(cols >> 3, 128));
}

// max|x| per segment into amax_ws (bf16 magnitude bits).  A tensor of at
// most 32 KB (decode-sized) is read by one CTA of 32 warps that stores the
// result, so the words need no clearing launch first; larger ones are cleared
// and reduced across the grid with atomics.
constexpr int64_t kOneBlockAmaxBytes = 32 * 1024;

int run_amax(DeviceState *d, const void *X, int64_t rows, int64_t K, int64_t ld, const nvfp4::SegRows &seg,
             uint32_t *amax_ws, cudaStream_t stream)
{
    if (rows > 0 && rows * K * 2 <= kOneBlockAmaxBytes) {
        const int64_t slices = std::max<int64_t>(amax_slices(rows, K), cdiv(32, rows));
        launch(nvfp4::amax_kernel, dim3(1), dim3(1024), 0, stream, static_cast<const uint16_t *>(X), rows, K, ld,
               slices, seg, amax_ws, d->status, static_cast<int32_t>(1));
        g_launches++;
        return launch_ok();
    }
    if (zero_words(amax_ws, seg.nseg, stream) != NVFP4_OK)
        return NVFP4_ERR_CUDA;
    if (rows > 0) {
        const int64_t slices = amax_slices(rows, K);
        const int64_t warps_needed = rows * slices;
        const int grid = static_cast<int>(std::min<int64_t>(cdiv(warps_needed, 8), int64_t(d->sm_count) * 8));
        launch(nvfp4::amax_kernel, dim3(grid), dim3(256), 0, stream, static_cast<const uint16_t *>(X), rows, K, ld,
               slices, seg, amax_ws, d->status, static_cast<int32_t>(0));
        g_launches++;
        return launch_ok();
    }
    return NVFP4_OK;
}

// The block quantizer: the single-segment kernel for activations (one global
// scale, rows in order), the general one for module segments or the gated
// row order.
void launch_quantize(const nvfp4::QuantParams &p, int grid, cudaStream_t stream)
{
    if (p.seg.nseg == 1 && p.gate_up_F == 0 && p.mode == 2)
        launch(nvfp4::quantize_act_kernel<true>, dim3(grid), dim3(256), 0, stream, p);
    else if (p.seg.nseg == 1 && p.gate_up_F == 0)
        launch(nvfp4::quantize_act_kernel<false>, dim3(grid), dim3(256), 0, stream, p);
    else
        launch(nvfp4::quantize_kernel, dim3(grid), dim3(256), 0, stream, p);
}

// K1 + K2 for `rows` x K bf16 rows, segment table `seg`.  mode 0: dynamic
// scale from max|x| (amax words in ws, g written to g_out); mode 1: scale
// read from g_in.
// zero_word, if given, is cleared by the quantize kernel (for the kernel that
// follows on the stream).
int run_quantize(DeviceState *d, const void *X, int64_t rows, int64_t K, int64_t ld, const nvfp4::SegRows &seg,
                 uint8_t *codes, uint8_t *sf, const float *g_in, float *g_out, bool dynamic, uint32_t *amax_ws,
                 cudaStream_t stream, int64_t gate_up_F = 0, uint32_t *zero_word = nullptr)
{
    const int64_t rows_pad = round_up(rows, 128);
    const int64_t groups = cdiv(K, 64);
    if (rows_pad * groups * 4 >= (int64_t(1) << 31) || K > (int64_t(1) << 30))
        return NVFP4_ERR_UNSUPPORTED_SHAPE;
    // a decode-sized activation (at most 32 KB): every quantize CTA takes
    // max|x| itself, one launch instead of the one-CTA amax pass and the
    // quantize (at 16 tokens, where every CTA would read 160-192 KB, that was
    // much slower)
    const bool cta_amax = dynamic && seg.nseg == 1 && gate_up_F == 0 && rows > 0 && rows * K * 2 <= kOneBlockAmaxBytes;
    if (dynamic && !cta_amax && run_amax(d, X, rows, K, ld, seg, amax_ws, stream) != NVFP4_OK)
        return NVFP4_ERR_CUDA;
    nvfp4::QuantParams p;
    p.X = static_cast<const uint16_t *>(X);
    p.ld = ld;
    p.rows = static_cast<int32_t>(rows);
    p.K = static_cast<int32_t>(K);
    p.rows_pad = static_cast<int32_t>(rows_pad);
    p.groups = static_cast<int32_t>(groups);
    p.seg = seg;
    p.amax_bits = amax_ws;
    p.g_in = g_in;
    p.g_out = g_out;
    p.mode = cta_amax ? 2 : (dynamic ? 0 : 1);
    p.status = d->status;
    p.codes = codes;
    p.sf = sf;
    p.gate_up_F = static_cast<int32_t>(gate_up_F);
    p.zero = zero_word;
    const int64_t threads = rows_pad * groups * 4;
    int grid = static_cast<int>(std::min<int64_t>(std::max<int64_t>(cdiv(threads, 256), 1), int64_t(d->sm_count) * 16));
    launch_quantize(p, grid, stream);
    g_launches++;
    return launch_ok();
}

// K2 alone for a contiguous [rows, K] bf16 matrix whose amax bits are already
// in amax_ws (one segment); writes codes, scales and g_out.
int run_quantize_from_amax(DeviceState *d, const void *X, int64_t rows, int64_t K, int64_t ld, const nvfp4::SegRows &seg,
                           uint8_t *codes, uint8_t *sf, float *g_out, const uint32_t *amax_ws, cudaStream_t stream)
{
    const int64_t rows_pad = round_up(rows, 128);
    const int64_t groups = cdiv(K, 64);
    if (rows_pad * groups * 4 >= (int64_t(1) << 31))
        return NVFP4_ERR_UNSUPPORTED_SHAPE;
    nvfp4::QuantParams p;
    p.X = static_cast<const uint16_t *>(X);
    p.ld = ld;
    p.rows = static_cast<int32_t>(rows);
    p.K = static_cast<int32_t>(K);
    p.rows_pad = static_cast<int32_t>(rows_pad);
    p.groups = static_cast<int32_t>(groups);
    p.seg = seg;
    p.amax_bits = amax_ws;
    p.g_in = nullptr;
    p.g_out = g_out;
    p.mode = 0;
    p.codes = codes;
    p.sf = sf;
    p.gate_up_F = 0;
    const int64_t threads = rows_pad * groups * 4;
    const int grid = static_cast<int>(std::min<int64_t>(std::max<int64_t>(cdiv(threads, 256), 1), int64_t(d->sm_count) * 16));
    launch_quantize(p, grid, stream);
    g_launches++;
    return launch_ok();
}

int make_codes_map(CUtensorMap *map, const uint8_t *codes, int64_t rows, int64_t K, uint32_t box_rows)
{
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(K / 2), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(K / 2)};
    cuuint32_t box[2] = {static_cast<cuuint32_t>(nvfp4::gemm::BK_BYTES), box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t *>(codes), dims, strides, box,
                          estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? NVFP4_OK : NVFP4_ERR_CUDA;
}

// Scale factors of a [rows, K] operand as a 2-D array of 8-byte elements:
// row = one 128-row tile, K/64 * 512 bytes long.  A box is one stage's
// 4 K-steps (2 KB; the whole row when K < 256) of box_rows row tiles.
int make_sf_map(CUtensorMap *map, const uint8_t *sf, int64_t row_tiles, int64_t kb_total, uint32_t box_rows,
                uint32_t *box_bytes)
{
    const int64_t inner = kb_total * 64;
    const uint32_t box_inner = static_cast<uint32_t>(std::min<int64_t>(inner, 256));
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(inner), static_cast<cuuint64_t>(row_tiles)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(kb_total * 512)};
    cuuint32_t box[2] = {box_inner, box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT64, 2, const_cast<uint8_t *>(sf), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    *box_bytes = box_inner * 8;
    return r == CUDA_SUCCESS ? NVFP4_OK : NVFP4_ERR_CUDA;
}

// bf16 output [rows, cols] as the TMA store target of the pair kernel's
// epilogue: 32-row x 64-column boxes, 128-byte swizzle.
int make_out_map(CUtensorMap *map, void *out, int64_t rows, int64_t cols)
{
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols * 2)};
    cuuint32_t box[2] = {64, 32};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, out, dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? NVFP4_OK : NVFP4_ERR_CUDA;
}

// Split-K for small M (one 128-row block): the single-CTA kernel has only
// cdiv(N, 256) output tiles there, too few to occupy 148 SMs, so each tile's
// K steps are divided into `splits` contiguous ranges that run as separate
// work items.  The count depends on the shape alone (sized for 148 SMs), so
// the result's bits do not depend on the device; every range is non-empty.
//
// The count minimises a cost model fitted to measurements on B200 at M <= 128:
// a CTA spends about 0.6 us per K stage (its pipeline is latency-bound at
// these sizes), while each split adds its fp32 partials (M x N x 4 bytes,
// written and read back by the finalize kernel) and a fixed cost for that
// kernel.  Below 64 rows the partials go out with per-row stores (about 1.5
// TB/s for the write and read together, 2 us fixed); from 64 rows the CTA's
// last work item stages them through shared memory, a row per store
// instruction (about 1.3 ns per partial element, 4.5 us fixed: fitted to
// split counts 1-8 at M = 64 and 128 on the decode shapes, N = 5120 with K
// = 5120, 6144, 17408 and N = 14432 with K = 5120).
constexpr int kSplitKMax = 8;
constexpr int kSplitKSms = 148;
constexpr int64_t kStagedPartialRows = 64;

int splitk_count(int64_t M, int64_t N, int64_t K)
{
    using namespace nvfp4::gemm;
    if (M <= 0 || M > BM || N <= 0 || K <= 0)
        return 1;
    const int64_t tiles = cdiv(N, BN);
    const int64_t kt_total = cdiv(K / 64, KB_PER_STAGE);
    const int64_t s_max = std::min<int64_t>({kSplitKMax, kt_total, std::max<int64_t>(1, kSplitKSms / tiles)});
    int64_t best = 1;
    double best_ns = 600.0 * static_cast<double>(kt_total);
    const bool staged = M >= kStagedPartialRows;
    for (int64_t want = 2; want <= s_max; ++want) {
        const int64_t kps = cdiv(kt_total, want);
        const int64_t S = cdiv(kt_total, kps);
        const double elems = static_cast<double>(S * M * N);
        const double ns = 600.0 * static_cast<double>(kps) + (staged ? elems * 1.3e-3 + 4500.0 : elems * 8.0 / 1500.0 + 2000.0);
        if (ns < best_ns) {
            best_ns = ns;
            best = S;
        }
    }
    return static_cast<int>(best);
}

// h_amax != nullptr selects the gated MLP epilogue (W is [gate | up]
// interleaved in 128-row blocks, N = 2F, out = h [M, F] bf16).  partial !=
// nullptr (room for splitk_count(M, N, K) fp32 [M, N] slices) lets a plain
// GEMM with M <= 128 split K; the splits are then summed in order by a
// second kernel.
int run_gemm(DeviceState *d, const uint8_t *a_codes, const uint8_t *a_sf, const float *g_a, int64_t M, int64_t K,
             const uint8_t *w_codes, const uint8_t *w_sf, int64_t N, const nvfp4::SegRows &seg, const float *g_w,
             void *out, unsigned flags, cudaStream_t stream, uint32_t *h_amax = nullptr, float *partial = nullptr,
             bool w_early = false)
{
    using namespace nvfp4::gemm;
    if (M == 0 || N == 0)
        return NVFP4_OK;
    // every operand is read by TMA, which needs 16-byte aligned bases (the
    // entry points check this already; internal callers pass workspace slices)
    if (!aligned16(a_codes) || !aligned16(w_codes) || !aligned16(a_sf) || !aligned16(w_sf))
        return NVFP4_ERR_MISALIGNED;
    const int64_t n_row_tiles = cdiv(N, 128);
    const uint32_t sfb_rows = n_row_tiles >= 2 ? 2u : 1u;
    CUtensorMap tmA, tmB, tmSFA, tmSFB;
    uint32_t sf_box = 0, sf_box_b = 0;
    // CTA pairs (256-row tiles) once A has more than one 128-row block
    const bool use_pair = (M > BM) && !(flags & NVFP4_SINGLE_CTA);
    // the single-CTA kernel loads only the rows a small M has (multiple of 8: one swizzle atom)
    const uint32_t a_rows = (!use_pair && M < BM) ? static_cast<uint32_t>(round_up(M, 8)) : static_cast<uint32_t>(BM);
    if (make_codes_map(&tmA, a_codes, M, K, a_rows) != NVFP4_OK ||
        make_codes_map(&tmB, w_codes, N, K, use_pair ? 128u : static_cast<uint32_t>(BN)) != NVFP4_OK ||
        make_sf_map(&tmSFA, a_sf, cdiv(M, 128), K / 64, 1, &sf_box) != NVFP4_OK ||
        make_sf_map(&tmSFB, w_sf, n_row_tiles, K / 64, sfb_rows, &sf_box_b) != NVFP4_OK)
        return NVFP4_ERR_CUDA;
    Params p;
    std::memset(&p, 0, sizeof(p));
    p.M = static_cast<int32_t>(M);
    p.N = static_cast<int32_t>(N);
    p.K = static_cast<int32_t>(K);
    p.num_m = static_cast<int32_t>(cdiv(M, BM));
    p.num_n = static_cast<int32_t>(cdiv(N, BN));
    p.num_tiles = p.num_m * p.num_n;
    p.a_box_bytes = a_rows * BK_BYTES;
    p.pair_m = static_cast<int32_t>(cdiv(M, pair::PAIR_M));
    p.pair_n = static_cast<int32_t>(cdiv(N, pair::PAIR_N));
    p.pair_tiles = p.pair_m * p.pair_n;
    p.kb_total = static_cast<int32_t>(K / 64);
    p.kt_total = static_cast<int32_t>(cdiv(K / 64, KB_PER_STAGE));
    p.splits = 1;
    p.kt_per_split = p.kt_total;
    if (partial != nullptr && h_amax == nullptr && !use_pair) {
        const int S = splitk_count(M, N, K);
        if (S > 1) {
            p.splits = S;
            p.kt_per_split = static_cast<int32_t>(cdiv(p.kt_total, S));
            p.partial = partial;
            p.staged_partials = M >= kStagedPartialRows ? 1 : 0;
        }
    }
    p.w_early = (w_early && !use_pair) ? 1 : 0;
    p.n_row_tiles = static_cast<int32_t>(n_row_tiles);
    p.sf_box_bytes = sf_box;
    p.sfb_box_rows = sfb_rows;
    p.sfa = a_sf;
    p.sfb = w_sf;
    p.g_a = g_a;
    p.g_w = g_w;
    p.nseg = seg.nseg;
    for (int i = 0; i < kMaxSeg; ++i)
        p.seg_end[i] = static_cast<int32_t>(seg.end[i]);
    p.out = out;
    p.out_fp32 = (flags & NVFP4_OUT_FP32) ? 1 : 0;
    const int64_t esz = p.out_fp32 ? 4 : 2;
    p.vec_ok = aligned16(out) && ((N * esz) % 16 == 0);
    p.status = d->status;
    // re-stream the smaller operand: A is M x K/2 bytes of codes, W is N x K/2
    p.n_fastest = (M > N) ? 1 : 0;
    p.inject_stall = (flags & NVFP4_DEBUG_INJECT_STALL) ? 1 : 0;
    p.wait_limit_ns = p.inject_stall ? 20000000ull : WAIT_LIMIT_NS;
    if (h_amax != nullptr) {
        p.F = static_cast<int32_t>(N / 2);
        p.h_amax = h_amax;
        p.vec_ok = aligned16(out) && ((p.F * 2) % 16 == 0);
    }
    if (use_pair) {
        // bf16 outputs with 16-byte rows leave through TMA stores
        CUtensorMap tmOut;
        std::memset(&tmOut, 0, sizeof(tmOut));
        p.tma_out = 0;
        if (!p.out_fp32 && p.vec_ok) {
            if (make_out_map(&tmOut, out, M, h_amax != nullptr ? N / 2 : N) != NVFP4_OK)
                return NVFP4_ERR_CUDA;
            p.tma_out = 1;
        }
        // one cluster of two CTAs per pair of SMs, persistent over the pair tiles
        const int grid = 2 * static_cast<int>(std::min<int64_t>(p.pair_tiles, d->sm_count / 2));
        if (h_amax != nullptr)
            launch(pair::gemm_nvf4_pair_kernel<true>, dim3(grid), dim3(pair::NUM_THREADS), pair::SMEM_BYTES, stream,
                   tmA, tmB, tmSFA, tmSFB, tmOut, p);
        else
            launch(pair::gemm_nvf4_pair_kernel<false>, dim3(grid), dim3(pair::NUM_THREADS), pair::SMEM_BYTES, stream,
                   tmA, tmB, tmSFA, tmSFB, tmOut, p);
    } else {
        const int grid = static_cast<int>(std::min<int64_t>(static_cast<int64_t>(p.num_tiles) * p.splits, d->sm_count));
        if (h_amax != nullptr)
            launch(gemm_nvf4_kernel<true>, dim3(grid), dim3(NUM_THREADS), SMEM_BYTES, stream, tmA, tmB, tmSFA, tmSFB, p);
        else
            launch(gemm_nvf4_kernel<false>, dim3(grid), dim3(NUM_THREADS), SMEM_BYTES, stream, tmA, tmB, tmSFA, tmSFB, p);
        if (p.splits > 1) {
            g_launches++;
            const int rc = launch_ok();
            if (rc != NVFP4_OK)
                return rc;
            const int64_t total = M * N;
            const int fin_grid = static_cast<int>(std::min<int64_t>(cdiv(total, 256), 4LL * d->sm_count));
            launch(splitk_finalize_kernel, dim3(fin_grid), dim3(256), 0, stream, static_cast<const float *>(partial),
                   p.splits, M, N, out, p.out_fp32);
        }
    }
    g_launches++;
    return launch_ok();
}

int check_gemm_shape(int64_t M, int64_t N, int64_t K)
{
    if (M < 0 || N < 0 || K <= 0)
        return NVFP4_ERR_INVALID_ARG;
    if (K % 64 != 0)
        return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (M > (int64_t(1) << 30) || N > (int64_t(1) << 30) || K > (int64_t(1) << 30) ||
        cdiv(M, nvfp4::gemm::BM) * cdiv(N, nvfp4::gemm::BN) >= (int64_t(1) << 31))
        return NVFP4_ERR_UNSUPPORTED_SHAPE;
    return NVFP4_OK;
}

constexpr size_t kLinScaleOff = 256;
constexpr size_t kLinHAmaxOff = 512;  // gated linear: max|h| word
constexpr size_t kLinCodesOff = 1024;

size_t linear_codes_bytes(int64_t M, int64_t K) { return static_cast<size_t>(M) * static_cast<size_t>(K / 2); }

size_t linear_sf_off(int64_t M, int64_t K)
{
    return static_cast<size_t>(round_up(static_cast<int64_t>(kLinCodesOff + linear_codes_bytes(M, K)), 1024));
}

// Split-K partial sums follow the activation's scale factors.
size_t linear_partial_off(int64_t M, int64_t K)
{
    return static_cast<size_t>(round_up(static_cast<int64_t>(linear_sf_off(M, K)) + sf_bytes_i(M, K), 256));
}

size_t linear_partial_bytes(int64_t M, int64_t N, int64_t K)
{
    const int S = splitk_count(M, N, K);
    return S > 1 ? static_cast<size_t>(S) * static_cast<size_t>(M) * static_cast<size_t>(N) * 4 : 0;
}

// nvfp4_gemm_prequant with an optional workspace for split-K partial sums
// (ws == nullptr: never split).
int gemm_prequant_impl(const uint8_t *a_codes, const uint8_t *a_sf, const float *g_a, int64_t M, int64_t K,
                       const uint8_t *w_codes, const uint8_t *w_sf, int64_t N, const nvfp4_segment *segs,
                       const float *g_w, int nseg, void *out, unsigned flags, void *ws, size_t ws_bytes,
                       void *stream)
{
    if ((flags & ~(NVFP4_STATIC_SCALE | NVFP4_OUT_FP32 | NVFP4_DEBUG_INJECT_STALL | NVFP4_SINGLE_CTA)) != 0)
        return NVFP4_ERR_INVALID_ARG;
    int rc = check_gemm_shape(M, N, K);
    if (rc != NVFP4_OK)
        return rc;
    {
        nvfp4::SegRows seg0;
        rc = check_segments(segs, nseg, N, &seg0);
        if (rc != NVFP4_OK)
            return rc;
    }
    if (M == 0 || N == 0)
        return NVFP4_OK;
    if (a_codes == nullptr || a_sf == nullptr || g_a == nullptr || w_codes == nullptr || w_sf == nullptr ||
        g_w == nullptr || out == nullptr)
        return NVFP4_ERR_INVALID_ARG;
    if (!aligned16(a_codes) || !aligned16(a_sf) || !aligned16(w_codes) || !aligned16(w_sf) ||
        (reinterpret_cast<uintptr_t>(g_a) & 3u) || (reinterpret_cast<uintptr_t>(g_w) & 3u) ||
        (reinterpret_cast<uintptr_t>(out) & ((flags & NVFP4_OUT_FP32) ? 3u : 1u)))
        return NVFP4_ERR_MISALIGNED;
    nvfp4::SegRows seg;
    rc = check_segments(segs, nseg, N, &seg);
    if (rc != NVFP4_OK)
        return rc;
    float *partial = nullptr;
    if (ws != nullptr) {
        const size_t need = linear_partial_bytes(M, N, K);
        if (ws_bytes < need)
            return NVFP4_ERR_WORKSPACE;
        if (!aligned16(ws))
            return NVFP4_ERR_MISALIGNED;
        if (need > 0)
            partial = static_cast<float *>(ws);
    }
    DeviceState *d = device_state();
    if (d == nullptr)
        return NVFP4_ERR_CUDA;
    if (!d->supported)
        return NVFP4_ERR_NO_DEVICE;
    return run_gemm(d, a_codes, a_sf, g_a, M, K, w_codes, w_sf, N, seg, g_w, out, flags,
                    static_cast<cudaStream_t>(stream), nullptr, partial);
}

}  // namespace

// ======================================================================== C ABI

extern "C" {

size_t nvfp4_sf_bytes(int64_t rows, int64_t K)
{
    if (rows < 0 || K <= 0 || K % 16 != 0)
        return 0;
    return static_cast<size_t>(sf_bytes_i(rows, K));
}

size_t nvfp4_quant_workspace_bytes(int nseg)
{
    if (nseg < 1 || nseg > kMaxSeg)
        return 0;
    return 256;
}

size_t nvfp4_workspace_bytes(int64_t M, int64_t N, int64_t K, int nseg)
{
    (void)nseg;
    if (M < 0 || N < 0 || K <= 0 || K % 16 != 0)
        return 0;
    const size_t partial = linear_partial_bytes(M, N, K);
    if (partial > 0)
        return linear_partial_off(M, K) + partial;
    return linear_sf_off(M, K) + static_cast<size_t>(sf_bytes_i(M, K));
}

size_t nvfp4_linear_act_scale_offset(void) { return kLinScaleOff; }

int nvfp4_quantize_weights(const void *W, int64_t N, int64_t K, int64_t ldw, const nvfp4_segment *segs, int nseg,
                           uint8_t *codes, uint8_t *sf, float *g_w, void *ws, size_t ws_bytes, void *stream)
{
    if (g_w == nullptr || N < 0 || K <= 0 || (N > 0 && (W == nullptr || codes == nullptr || sf == nullptr)))
        return NVFP4_ERR_INVALID_ARG;
    if (K % 16 != 0)
        return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (ldw < K)
        return NVFP4_ERR_INVALID_ARG;
    if (!aligned16(W) || ldw % 8 != 0 || !aligned16(codes) || !aligned16(sf))
        return NVFP4_ERR_MISALIGNED;
    nvfp4::SegRows seg;
    int rc = check_segments(segs, nseg, N, &seg);
    if (rc != NVFP4_OK)
        return rc;
    if (ws == nullptr || ws_bytes < nvfp4_quant_workspace_bytes(nseg))
        return NVFP4_ERR_WORKSPACE;
    DeviceState *d = device_state();
    if (d == nullptr)
        return NVFP4_ERR_CUDA;
    if (!d->supported)
        return NVFP4_ERR_NO_DEVICE;
    return run_quantize(d, W, N, K, ldw, seg, codes, sf, nullptr, g_w, true, static_cast<uint32_t *>(ws),
                        static_cast<cudaStream_t>(stream));
}

int nvfp4_quantize_act(const void *X, int64_t M, int64_t K, int64_t ldx, uint8_t *codes, uint8_t *sf, float *g_a,
                       unsigned flags, void *ws, size_t ws_bytes, void *stream)
{
    if (g_a == nullptr || M < 0 || K <= 0 || (M > 0 && (X == nullptr || codes == nullptr || sf == nullptr)))
        return NVFP4_ERR_INVALID_ARG;
    if ((flags & ~(NVFP4_STATIC_SCALE | NVFP4_OUT_FP32 | NVFP4_AMAX_GIVEN)) != 0 ||
        ((flags & NVFP4_STATIC_SCALE) && (flags & NVFP4_AMAX_GIVEN)))
        return NVFP4_ERR_INVALID_ARG;
    if (K % 16 != 0)
        return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (ldx < K)
        return NVFP4_ERR_INVALID_ARG;
    if (!aligned16(X) || ldx % 8 != 0 || !aligned16(codes) || !aligned16(sf) ||
        (reinterpret_cast<uintptr_t>(g_a) & 3u))
        return NVFP4_ERR_MISALIGNED;
    const bool dynamic = (flags & NVFP4_STATIC_SCALE) == 0;
    if (dynamic && (ws == nullptr || ws_bytes < nvfp4_quant_workspace_bytes(1)))
        return NVFP4_ERR_WORKSPACE;
    DeviceState *d = device_state();
    if (d == nullptr)
        return NVFP4_ERR_CUDA;
    if (!d->supported)
        return NVFP4_ERR_NO_DEVICE;
    nvfp4::SegRows seg;
    nvfp4_segment one = {0, M};
    check_segments(&one, 1, M, &seg);
    if (flags & NVFP4_AMAX_GIVEN)
        return run_quantize_from_amax(d, X, M, K, ldx, seg, codes, sf, g_a, static_cast<const uint32_t *>(ws),
                                      static_cast<cudaStream_t>(stream));
    return run_quantize(d, X, M, K, ldx, seg, codes, sf, g_a, g_a, dynamic, static_cast<uint32_t *>(ws),
                        static_cast<cudaStream_t>(stream));
}

int nvfp4_gemm_prequant(const uint8_t *a_codes, const uint8_t *a_sf, const float *g_a, int64_t M, int64_t K,
                        const uint8_t *w_codes, const uint8_t *w_sf, int64_t N, const nvfp4_segment *segs,
                        const float *g_w, int nseg, void *out, unsigned flags, void *stream)
{
    return gemm_prequant_impl(a_codes, a_sf, g_a, M, K, w_codes, w_sf, N, segs, g_w, nseg, out, flags, nullptr, 0,
                              stream);
}

size_t nvfp4_gemm_workspace_bytes(int64_t M, int64_t N, int64_t K)
{
    if (M < 0 || N < 0 || K <= 0 || K % 64 != 0)
        return 0;
    return linear_partial_bytes(M, N, K);
}

int nvfp4_gemm_prequant_ws(const uint8_t *a_codes, const uint8_t *a_sf, const float *g_a, int64_t M, int64_t K,
                           const uint8_t *w_codes, const uint8_t *w_sf, int64_t N, const nvfp4_segment *segs,
                           const float *g_w, int nseg, void *out, unsigned flags, void *ws, size_t ws_bytes,
                           void *stream)
{
    return gemm_prequant_impl(a_codes, a_sf, g_a, M, K, w_codes, w_sf, N, segs, g_w, nseg, out, flags, ws, ws_bytes,
                              stream);
}

int nvfp4_linear_fused(const void *X, int64_t M, int64_t K, const uint8_t *w_codes, const uint8_t *w_sf, int64_t N,
                       const nvfp4_segment *segs, const float *g_w, int nseg, void *out, unsigned flags, void *ws,
                       size_t ws_bytes, void *stream)
{
    if ((flags & ~(NVFP4_STATIC_SCALE | NVFP4_OUT_FP32 | NVFP4_SINGLE_CTA)) != 0)
        return NVFP4_ERR_INVALID_ARG;
    int rc = check_gemm_shape(M, N, K);
    if (rc != NVFP4_OK)
        return rc;
    {
        nvfp4::SegRows seg0;
        rc = check_segments(segs, nseg, N, &seg0);
        if (rc != NVFP4_OK)
            return rc;
    }
    if (M == 0 || N == 0)
        return NVFP4_OK;
    if (X == nullptr || w_codes == nullptr || w_sf == nullptr || g_w == nullptr || out == nullptr)
        return NVFP4_ERR_INVALID_ARG;
    if (!aligned16(X) || K % 8 != 0 || !aligned16(w_codes) || !aligned16(w_sf) ||
        (reinterpret_cast<uintptr_t>(g_w) & 3u) ||
        (reinterpret_cast<uintptr_t>(out) & ((flags & NVFP4_OUT_FP32) ? 3u : 1u)))
        return NVFP4_ERR_MISALIGNED;
    nvfp4::SegRows seg;
    rc = check_segments(segs, nseg, N, &seg);
    if (rc != NVFP4_OK)
        return rc;
    if (ws == nullptr || !aligned16(ws) || ws_bytes < nvfp4_workspace_bytes(M, N, K, nseg))
        return NVFP4_ERR_WORKSPACE;
    DeviceState *d = device_state();
    if (d == nullptr)
        return NVFP4_ERR_CUDA;
    if (!d->supported)
        return NVFP4_ERR_NO_DEVICE;
    uint8_t *base = static_cast<uint8_t *>(ws);
    uint32_t *amax = reinterpret_cast<uint32_t *>(base);
    float *g_a = reinterpret_cast<float *>(base + kLinScaleOff);
    uint8_t *a_codes = base + kLinCodesOff;
    uint8_t *a_sf = base + linear_sf_off(M, K);
    nvfp4::SegRows one_seg;
    nvfp4_segment one = {0, M};
    check_segments(&one, 1, M, &one_seg);
    const bool dynamic = (flags & NVFP4_STATIC_SCALE) == 0;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    float *partial =
        linear_partial_bytes(M, N, K) > 0 ? reinterpret_cast<float *>(base + linear_partial_off(M, K)) : nullptr;
    rc = run_quantize(d, X, M, K, K, one_seg, a_codes, a_sf, g_a, g_a, dynamic, amax, s);
    if (rc != NVFP4_OK)
        return rc;
    // the GEMM follows this call's own quantize kernel, which does not write W
    return run_gemm(d, a_codes, a_sf, g_a, M, K, w_codes, w_sf, N, seg, g_w, out, flags, s, nullptr, partial, true);
}

int nvfp4_linear(const void *X, int64_t M, int64_t K, const uint8_t *w_codes, const uint8_t *w_sf, const float *g_w,
                 int64_t N, void *out, unsigned flags, void *ws, size_t ws_bytes, void *stream)
{
    if (N < 0)
        return NVFP4_ERR_INVALID_ARG;
    nvfp4_segment one = {0, N};
    return nvfp4_linear_fused(X, M, K, w_codes, w_sf, N, &one, g_w, 1, out, flags, ws, ws_bytes, stream);
}

int nvfp4_swiglu_quantize(const void *gate_up, int64_t M, int64_t F, int64_t ld, void *h, uint8_t *codes, uint8_t *sf,
                          float *g_h, void *ws, size_t ws_bytes, void *stream)
{
    if (gate_up == nullptr || h == nullptr || codes == nullptr || sf == nullptr || g_h == nullptr || M < 0 || F <= 0)
        return NVFP4_ERR_INVALID_ARG;
    if (F % 16 != 0)
        return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (ld < 2 * F)
        return NVFP4_ERR_INVALID_ARG;
    if (!aligned16(gate_up) || ld % 8 != 0 || !aligned16(h) || !aligned16(codes) || !aligned16(sf))
        return NVFP4_ERR_MISALIGNED;
    if (ws == nullptr || ws_bytes < nvfp4_quant_workspace_bytes(1))
        return NVFP4_ERR_WORKSPACE;
    if (M * (F / 8) >= (int64_t(1) << 31))
        return NVFP4_ERR_UNSUPPORTED_SHAPE;
    DeviceState *d = device_state();
    if (d == nullptr)
        return NVFP4_ERR_CUDA;
    if (!d->supported)
        return NVFP4_ERR_NO_DEVICE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint32_t *amax = static_cast<uint32_t *>(ws);
    if (zero_words(amax, 1, s) != NVFP4_OK)
        return NVFP4_ERR_CUDA;
    if (M > 0) {
        const int64_t threads = M * (F / 8);
        const int grid = static_cast<int>(std::min<int64_t>(cdiv(threads, 256), int64_t(d->sm_count) * 16));
        launch(nvfp4::swiglu_kernel, dim3(grid), dim3(256), 0, s, static_cast<const uint16_t *>(gate_up), ld,
               static_cast<int32_t>(M), static_cast<int32_t>(F), static_cast<uint16_t *>(h), amax);
        g_launches++;
        if (launch_ok() != NVFP4_OK)
            return NVFP4_ERR_CUDA;
    }
    nvfp4::SegRows seg;
    nvfp4_segment one = {0, M};
    check_segments(&one, 1, M, &seg);
    // the amax of h was folded in by the SwiGLU kernel: quantize without a new amax pass
    const int64_t rows_pad = round_up(M, 128);
    const int64_t groups = cdiv(F, 64);
    if (rows_pad * groups * 4 >= (int64_t(1) << 31))
        return NVFP4_ERR_UNSUPPORTED_SHAPE;
    nvfp4::QuantParams p;
    p.X = static_cast<const uint16_t *>(h);
    p.ld = F;
    p.rows = static_cast<int32_t>(M);
    p.K = static_cast<int32_t>(F);
    p.rows_pad = static_cast<int32_t>(rows_pad);
    p.groups = static_cast<int32_t>(groups);
    p.seg = seg;
    p.amax_bits = amax;
    p.g_in = nullptr;
    p.g_out = g_h;
    p.mode = 0;
    p.codes = codes;
    p.sf = sf;
    p.gate_up_F = 0;
    const int64_t threads = rows_pad * groups * 4;
    const int grid = static_cast<int>(std::min<int64_t>(std::max<int64_t>(cdiv(threads, 256), 1), int64_t(d->sm_count) * 16));
    launch_quantize(p, grid, s);
    g_launches++;
    return launch_ok();
}

int nvfp4_get_status(void *stream)
{
    DeviceState *d = device_state();
    if (d == nullptr)
        return NVFP4_ERR_CUDA;
    if (!d->supported)
        return NVFP4_ERR_NO_DEVICE;
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess)
        return NVFP4_ERR_CUDA;
    uint32_t v = 0;
    if (cudaMemcpy(&v, d->status, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess)
        return NVFP4_ERR_CUDA;
    const uint32_t zero = 0;
    if (cudaMemcpy(d->status, &zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess)
        return NVFP4_ERR_CUDA;
    if (v & nvfp4::kStatusTimeout)
        return NVFP4_ERR_TIMEOUT;
    if (v & nvfp4::kStatusNonFinite)
        return NVFP4_ERR_NONFINITE;
    return NVFP4_OK;
}

const char *nvfp4_status_string(int status)
{
    switch (status) {
    case NVFP4_OK: return "ok";
    case NVFP4_ERR_INVALID_ARG: return "invalid argument";
    case NVFP4_ERR_UNSUPPORTED_SHAPE: return "unsupported shape (K must be a multiple of 16, 64 for GEMMs)";
    case NVFP4_ERR_MISALIGNED: return "misaligned pointer or leading dimension";
    case NVFP4_ERR_CUDA: return "CUDA runtime error";
    case NVFP4_ERR_TIMEOUT: return "a bounded wait inside a kernel ran out";
    case NVFP4_ERR_NONFINITE: return "input contains Inf or NaN";
    case NVFP4_ERR_WORKSPACE: return "workspace missing or too small";
    case NVFP4_ERR_NO_DEVICE: return "current device is not an sm_100 GPU";
    default: return "unknown status";
    }
}

int nvfp4_device_supported(void)
{
    DeviceState *d = device_state();
    return (d != nullptr && d->supported) ? 1 : 0;
}

uint64_t nvfp4_launch_count(void) { return g_launches.load(); }

}  // extern "C"

// ------------------------------------------------- allocation-free linear

namespace {

// Scratch of nvfp4_linear_fused_noalloc, laid out like a linear workspace:
// [amax word | g_a | activation codes | activation scale factors].
constexpr size_t kNoAllocCodesBytes = static_cast<size_t>(NVFP4_NOALLOC_MAX_ELEMS) / 2;
constexpr size_t kNoAllocSfOff = kLinCodesOff + kNoAllocCodesBytes;
constexpr size_t kNoAllocBytes = kNoAllocSfOff + static_cast<size_t>(NVFP4_NOALLOC_MAX_SF_BYTES);
static_assert(kNoAllocSfOff % 1024 == 0, "scale factors must stay 16-byte aligned for the bulk copies");

static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocBytes];

// Device address of g_noalloc_scratch per device (the host-side symbol is a
// stand-in, never a device pointer).  Written once per device under the
// mutex (release), read without it (acquire).
std::atomic<uint8_t *> g_noalloc_ptr[kMaxDevices] = {};
std::mutex g_noalloc_mu;

uint8_t *noalloc_scratch()
{
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
        return nullptr;
    uint8_t *known = g_noalloc_ptr[dev].load(std::memory_order_acquire);
    if (known != nullptr)
        return known;
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    known = g_noalloc_ptr[dev].load(std::memory_order_relaxed);
    if (known == nullptr) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
            return nullptr;
        known = static_cast<uint8_t *>(p);
        g_noalloc_ptr[dev].store(known, std::memory_order_release);
    }
    return known;
}

}  // namespace

extern "C" int nvfp4_linear_fused_noalloc(const void *X, int64_t M, int64_t K, const uint8_t *w_codes,
                                          const uint8_t *w_sf, int64_t N, const nvfp4_segment *segs,
                                          const float *g_w, int nseg, void *out, unsigned flags, void *stream)
{
    if ((flags & ~static_cast<unsigned>(NVFP4_OUT_FP32)) != 0)
        return NVFP4_ERR_INVALID_ARG;
    int rc = check_gemm_shape(M, N, K);
    if (rc != NVFP4_OK)
        return rc;
    nvfp4::SegRows seg;
    rc = check_segments(segs, nseg, N, &seg);
    if (rc != NVFP4_OK)
        return rc;
    if (M * K > NVFP4_NOALLOC_MAX_ELEMS || sf_bytes_i(M, K) > NVFP4_NOALLOC_MAX_SF_BYTES)
        return NVFP4_ERR_WORKSPACE;
    if (M == 0 || N == 0)
        return NVFP4_OK;
    if (X == nullptr || w_codes == nullptr || w_sf == nullptr || g_w == nullptr || out == nullptr)
        return NVFP4_ERR_INVALID_ARG;
    if (!aligned16(X) || K % 8 != 0 || !aligned16(w_codes) || !aligned16(w_sf) ||
        (reinterpret_cast<uintptr_t>(g_w) & 3u) ||
        (reinterpret_cast<uintptr_t>(out) & ((flags & NVFP4_OUT_FP32) ? 3u : 1u)))
        return NVFP4_ERR_MISALIGNED;
    DeviceState *d = device_state();
    if (d == nullptr)
        return NVFP4_ERR_CUDA;
    if (!d->supported)
        return NVFP4_ERR_NO_DEVICE;
    uint8_t *base = noalloc_scratch();
    if (base == nullptr)
        return NVFP4_ERR_CUDA;
    uint32_t *amax = reinterpret_cast<uint32_t *>(base);
    float *g_a = reinterpret_cast<float *>(base + kLinScaleOff);
    uint8_t *a_codes = base + kLinCodesOff;
    uint8_t *a_sf = base + kNoAllocSfOff;
    nvfp4::SegRows one_seg;
    nvfp4_segment one = {0, M};
    check_segments(&one, 1, M, &one_seg);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    rc = run_quantize(d, X, M, K, K, one_seg, a_codes, a_sf, g_a, g_a, true, amax, s);
    if (rc != NVFP4_OK)
        return rc;
    // the GEMM follows this call's own quantize kernel, which does not write W
    return run_gemm(d, a_codes, a_sf, g_a, M, K, w_codes, w_sf, N, seg, g_w, out, flags, s, nullptr, nullptr, true);
}

// ------------------------------------------------------ gated MLP (SwiGLU)

extern "C" int nvfp4_quantize_weights_gated(const void *W, int64_t F, int64_t K, int64_t ldw, uint8_t *codes,
                                            uint8_t *sf, float *g_w, void *ws, size_t ws_bytes, void *stream)
{
    if (W == nullptr || codes == nullptr || sf == nullptr || g_w == nullptr || F <= 0 || K <= 0)
        return NVFP4_ERR_INVALID_ARG;
    if (K % 16 != 0 || F % 128 != 0)
        return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (ldw < K)
        return NVFP4_ERR_INVALID_ARG;
    if (!aligned16(W) || ldw % 8 != 0 || !aligned16(codes) || !aligned16(sf))
        return NVFP4_ERR_MISALIGNED;
    if (ws == nullptr || ws_bytes < nvfp4_quant_workspace_bytes(2))
        return NVFP4_ERR_WORKSPACE;
    DeviceState *d = device_state();
    if (d == nullptr)
        return NVFP4_ERR_CUDA;
    if (!d->supported)
        return NVFP4_ERR_NO_DEVICE;
    nvfp4::SegRows seg;
    const nvfp4_segment two[2] = {{0, F}, {F, 2 * F}};
    check_segments(two, 2, 2 * F, &seg);
    return run_quantize(d, W, 2 * F, K, ldw, seg, codes, sf, nullptr, g_w, true, static_cast<uint32_t *>(ws),
                        static_cast<cudaStream_t>(stream), F);
}

extern "C" int nvfp4_gemm_prequant_swiglu(const uint8_t *a_codes, const uint8_t *a_sf, const float *g_a, int64_t M,
                                          int64_t K, const uint8_t *w_codes, const uint8_t *w_sf, int64_t F,
                                          const float *g_w, void *h, void *ws, size_t ws_bytes, void *stream)
{
    int rc = check_gemm_shape(M, 2 * F, K);
    if (rc != NVFP4_OK)
        return rc;
    if (F <= 0)
        return NVFP4_ERR_INVALID_ARG;
    if (F % 128 != 0)
        return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (ws == nullptr || ws_bytes < nvfp4_quant_workspace_bytes(1))
        return NVFP4_ERR_WORKSPACE;
    if (M > 0 && (a_codes == nullptr || a_sf == nullptr || g_a == nullptr || w_codes == nullptr ||
                  w_sf == nullptr || g_w == nullptr || h == nullptr))
        return NVFP4_ERR_INVALID_ARG;
    if (!aligned16(a_codes) || !aligned16(a_sf) || !aligned16(w_codes) || !aligned16(w_sf) || !aligned16(h) ||
        !aligned16(ws) || (reinterpret_cast<uintptr_t>(g_a) & 3u) || (reinterpret_cast<uintptr_t>(g_w) & 3u))
        return NVFP4_ERR_MISALIGNED;
    DeviceState *d = device_state();
    if (d == nullptr)
        return NVFP4_ERR_CUDA;
    if (!d->supported)
        return NVFP4_ERR_NO_DEVICE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint32_t *h_amax = static_cast<uint32_t *>(ws);
    if (zero_words(h_amax, 1, s) != NVFP4_OK)
        return NVFP4_ERR_CUDA;
    nvfp4::SegRows gu;
    const nvfp4_segment two[2] = {{0, F}, {F, 2 * F}};
    check_segments(two, 2, 2 * F, &gu);
    // the GEMM follows this call's own clearing of h_amax, which does not write W
    return run_gemm(d, a_codes, a_sf, g_a, M, K, w_codes, w_sf, 2 * F, gu, g_w, h, 0, s, h_amax, nullptr, true);
}

extern "C" int nvfp4_linear_swiglu(const void *X, int64_t M, int64_t K, const uint8_t *w_codes, const uint8_t *w_sf,
                                   int64_t F, const float *g_w, void *h, uint8_t *h_codes, uint8_t *h_sf, float *g_h,
                                   unsigned flags, void *ws, size_t ws_bytes, void *stream)
{
    if ((flags & ~(NVFP4_STATIC_SCALE | NVFP4_SINGLE_CTA)) != 0)
        return NVFP4_ERR_INVALID_ARG;
    int rc = check_gemm_shape(M, 2 * F, K);
    if (rc != NVFP4_OK)
        return rc;
    if (F <= 0)
        return NVFP4_ERR_INVALID_ARG;
    if (F % 128 != 0)
        return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (g_h == nullptr || (M > 0 && (X == nullptr || w_codes == nullptr || w_sf == nullptr || g_w == nullptr ||
                                     h == nullptr || h_codes == nullptr || h_sf == nullptr)))
        return NVFP4_ERR_INVALID_ARG;
    if (!aligned16(X) || K % 8 != 0 || !aligned16(w_codes) || !aligned16(w_sf) || !aligned16(h) ||
        !aligned16(h_codes) || !aligned16(h_sf) || (reinterpret_cast<uintptr_t>(g_w) & 3u) ||
        (reinterpret_cast<uintptr_t>(g_h) & 3u))
        return NVFP4_ERR_MISALIGNED;
    if (ws == nullptr || !aligned16(ws) || ws_bytes < nvfp4_workspace_bytes(M, 2 * F, K, 2))
        return NVFP4_ERR_WORKSPACE;
    DeviceState *d = device_state();
    if (d == nullptr)
        return NVFP4_ERR_CUDA;
    if (!d->supported)
        return NVFP4_ERR_NO_DEVICE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint8_t *base = static_cast<uint8_t *>(ws);
    uint32_t *amax = reinterpret_cast<uint32_t *>(base);
    float *g_a = reinterpret_cast<float *>(base + kLinScaleOff);
    uint32_t *h_amax = reinterpret_cast<uint32_t *>(base + kLinHAmaxOff);
    uint8_t *a_codes = base + kLinCodesOff;
    uint8_t *a_sf = base + linear_sf_off(M, K);
    nvfp4::SegRows one_seg;
    nvfp4_segment one = {0, M};
    check_segments(&one, 1, M, &one_seg);
    // X -> NVFP4 (dynamic scale unless a calibrated one is supplied); the
    // quantize kernel also clears max|h| for the GEMM's epilogue
    rc = run_quantize(d, X, M, K, K, one_seg, a_codes, a_sf, g_a, g_a, (flags & NVFP4_STATIC_SCALE) == 0, amax, s, 0,
                      h_amax);
    if (rc != NVFP4_OK)
        return rc;
    // gate/up GEMM with the SwiGLU epilogue -> h (bf16) and max|h|
    nvfp4::SegRows gu;
    const nvfp4_segment two[2] = {{0, F}, {F, 2 * F}};
    check_segments(two, 2, 2 * F, &gu);
    // the GEMM follows this call's own quantize kernel, which does not write W
    rc = run_gemm(d, a_codes, a_sf, g_a, M, K, w_codes, w_sf, 2 * F, gu, g_w, h, flags & NVFP4_SINGLE_CTA, s, h_amax,
                  nullptr, true);
    if (rc != NVFP4_OK)
        return rc;
    // h -> NVFP4 with the dynamic scale folded in by the epilogue
    return run_quantize_from_amax(d, h, M, F, F, one_seg, h_codes, h_sf, g_h, h_amax, s);
}

// ------------------------------------------------- FP8 KV-cache (E4M3)

namespace {

int check_kv_shape(const void *X, int64_t rows, int64_t cols, int64_t ldx)
{
    if (rows < 0 || cols < 0 || ldx < cols || (rows > 0 && cols > 0 && X == nullptr))
        return NVFP4_ERR_INVALID_ARG;
    if (cols % 8 != 0)
        return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(X) || ldx % 8 != 0)
        return NVFP4_ERR_MISALIGNED;
    return NVFP4_OK;
}

}  // namespace

extern "C" int nvfp4_fp8_kv_calibrate(const void *X, int64_t rows, int64_t cols, int64_t ldx, float *scale, void *ws,
                                      size_t ws_bytes, void *stream)
{
    int rc = check_kv_shape(X, rows, cols, ldx);
    if (rc != NVFP4_OK)
        return rc;
    if (scale == nullptr)
        return NVFP4_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(scale) & 3u)
        return NVFP4_ERR_MISALIGNED;
    if (ws == nullptr || ws_bytes < nvfp4_quant_workspace_bytes(1) || (reinterpret_cast<uintptr_t>(ws) & 3u))
        return NVFP4_ERR_WORKSPACE;
    DeviceState *d = device_state();
    if (d == nullptr)
        return NVFP4_ERR_CUDA;
    if (!d->supported)
        return NVFP4_ERR_NO_DEVICE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint32_t *amax = static_cast<uint32_t *>(ws);
    nvfp4::SegRows seg;
    nvfp4_segment one = {0, std::max<int64_t>(rows, 1)};
    check_segments(&one, 1, std::max<int64_t>(rows, 1), &seg);
    if (run_amax(d, X, cols > 0 ? rows : 0, cols, ldx, seg, amax, s) != NVFP4_OK)
        return NVFP4_ERR_CUDA;
    launch(nvfp4::kv::kv_scale_kernel, dim3(1), dim3(32), 0, s, amax, scale);
    g_launches++;
    return launch_ok();
}

extern "C" int nvfp4_fp8_kv_quantize(const void *X, int64_t rows, int64_t cols, int64_t ldx, const float *scale,
                                     uint8_t *out, int64_t ldo, void *stream)
{
    int rc = check_kv_shape(X, rows, cols, ldx);
    if (rc != NVFP4_OK)
        return rc;
    if (scale == nullptr || ldo < cols || (rows > 0 && cols > 0 && out == nullptr))
        return NVFP4_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(scale) & 3u) || (reinterpret_cast<uintptr_t>(out) & 7u) || ldo % 8 != 0)
        return NVFP4_ERR_MISALIGNED;
    if (rows == 0 || cols == 0)
        return NVFP4_OK;
    DeviceState *d = device_state();
    if (d == nullptr)
        return NVFP4_ERR_CUDA;
    if (!d->supported)
        return NVFP4_ERR_NO_DEVICE;
    nvfp4::kv::KvParams p;
    p.X = static_cast<const uint16_t *>(X);
    p.ld = ldx;
    p.rows = rows;
    p.cols = cols;
    p.scale = scale;
    p.out = out;
    p.ldo = ldo;
    p.status = d->status;
    const int64_t groups = rows * (cols / 8);
    const int grid = static_cast<int>(std::min<int64_t>(cdiv(groups, 256), int64_t(d->sm_count) * 16));
    launch(nvfp4::kv::kv_quantize_kernel, dim3(grid), dim3(256), 0, static_cast<cudaStream_t>(stream), p);
    g_launches++;
    return launch_ok();
}
