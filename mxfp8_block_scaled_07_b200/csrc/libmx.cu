// libmx: the C-ABI entry points declared in include/mx.h. Host-side argument checks, tensor-map
// construction and kernel launches; the kernels themselves are in quantize.cuh, grid_equal.cuh
// and gemm.cuh. Nothing here allocates device memory or synchronizes (except mx_device_error).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <unordered_map>

#include "../../include/mx.h"
#include "blockwise.cuh"
#include "gemm.cuh"
#include "grid_equal.cuh"
#include "ptx.cuh"
#include "quantize.cuh"
#include "quantize_tma.cuh"
#include "swizzle.cuh"

namespace mx {

// Device status word: error bits set by kernels (expired bounded waits, bad grouped offsets).
__device__ uint32_t g_status_word;

__global__ void expired_wait_kernel(uint32_t* err, uint64_t timeout_ns) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort_flag = 0;
        fence_barrier_init();
    }
    __syncthreads();
    // Nothing arrives on `bar`: the wait must expire, record the error and return.
    mbar_wait(&bar, 0, reinterpret_cast<volatile int*>(&abort_flag), err, timeout_ns);
}

namespace {

constexpr int kMaxDevices = 64;
constexpr uint64_t kDefaultTimeoutNs = 2000000000ull;
std::atomic<uint64_t> g_timeout_ns{kDefaultTimeoutNs};

struct DeviceInfo {
    int sms = 0;
    int cc_major = 0;
    uint32_t* status = nullptr;
    int quant_blocks_per_sm[4] = {0, 0, 0, 0};
    int qt_blocks_per_sm[4] = {0, 0, 0, 0};   // TMA-staged quantizer, by direction bits
    int ge_blocks_per_sm = 1;
    int pair_clusters[2] = {0, 0};    // co-resident 2-CTA clusters of the pair GEMM (dense, grouped)
    bool ok = false;
};

// Clusters of 2 CTAs of `kernel` that fit on the device at once (falls back to SMs / 2).
template <class K>
int max_pair_clusters(K kernel, int smem, int sms) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2, 1, 1);
    cfg.blockDim = dim3(kGemmThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kernel, &cfg) != cudaSuccess || n < 1) {
        cudaGetLastError();
        n = sms / 2;
    }
    return n;
}

// GEMM kernel selection: 0 = CTA-pair kernel (default), 1 = single-CTA kernel.
std::atomic<int> g_gemm_variant{0};
// Quantizer selection: 0 = register-staged tiles (default; columnwise-only calls take the TMA-staged
// kernel, measured faster for that direction; rowwise-only calls whose CTAs each walk at least
// kSplitTilesPerCta tiles take the split-load form), 1 = TMA-staged tiles, 2 = as 0 with the
// split-load form for every rowwise-only call.
constexpr int64_t kSplitTilesPerCta = 64;
std::atomic<int> g_quant_variant{0};

bool use_tma_quantizer(bool row, bool col) { return g_quant_variant.load() == 1 || (col && !row); }
DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mutex;

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;
std::once_flag g_encode_once;

template <bool ROW>
int quant_occupancy() {
    int n = 0;
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, quantize_rowcol_kernel<ROW, kQMaxTensors>, kQThreads, 0);
    return n > 0 ? n : 1;
}

// Opts the TMA-staged quantizer (both tensor-count instantiations) into its dynamic shared memory
// and returns its resident CTAs per SM.
template <bool ROW, bool COL>
bool qt_setup(int* blocks) {
    if (cudaFuncSetAttribute(quantize_tma_kernel<ROW, COL, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kQtSmemBytes) != cudaSuccess ||
        cudaFuncSetAttribute(quantize_tma_kernel<ROW, COL, kQtMaxTensors>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, kQtSmemBytes) != cudaSuccess)
        return false;
    int n = 0;
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, quantize_tma_kernel<ROW, COL, kQtMaxTensors>, kQThreads,
                                                  kQtSmemBytes);
    *blocks = n > 0 ? n : 1;
    return true;
}

// Per-device facts, queried once with that device current.
const DeviceInfo* device_info() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(g_dev_mutex);
    DeviceInfo& d = g_dev[dev];
    if (!d.ok) {
        if (cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return nullptr;
        if (cudaDeviceGetAttribute(&d.cc_major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
            return nullptr;
        if (d.cc_major != 10) {
            d.ok = true;   // remembered as unsupported
            return &d;
        }
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_status_word) != cudaSuccess) return nullptr;
        d.status = static_cast<uint32_t*>(p);
        // Resident CTAs of the rowwise kernel: the smallest over its load schedules and the fused
        // comparison forms, which all launch with this grid.
        int blocks[3] = {0, 0, 0};
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&d.quant_blocks_per_sm[1],
                                                      quantize_rowwise_kernel<kQMaxTensors, false>, kQThreads, 0);
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&blocks[0], quantize_rowwise_kernel<kQMaxTensors, true>,
                                                      kQThreads, 0);
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&blocks[1], quantize_rowwise_kernel<kQMaxTensors, false, true>,
                                                      kQThreads, 0);
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&blocks[2], quantize_rowwise_kernel<kQMaxTensors, true, true>,
                                                      kQThreads, 0);
        for (int b : blocks) d.quant_blocks_per_sm[1] = std::min(d.quant_blocks_per_sm[1], b);
        if (d.quant_blocks_per_sm[1] < 1) d.quant_blocks_per_sm[1] = 1;
        d.quant_blocks_per_sm[3] = quant_occupancy<true>();
        if (!qt_setup<true, false>(&d.qt_blocks_per_sm[1]) || !qt_setup<false, true>(&d.qt_blocks_per_sm[2]) ||
            !qt_setup<true, true>(&d.qt_blocks_per_sm[3]))
            return nullptr;
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&d.ge_blocks_per_sm, grid_equal_kernel<kGeMaxPairs>,
                                                      kGeThreads, 0);
        if (d.ge_blocks_per_sm < 1) d.ge_blocks_per_sm = 1;
        if (cudaFuncSetAttribute(mx_gemm_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 kGemmSmemDense) != cudaSuccess ||
            cudaFuncSetAttribute(mx_gemm_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 kGemmSmemGrouped) != cudaSuccess ||
            cudaFuncSetAttribute(mx_gemm_pair_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 kGemmPairSmemDense) != cudaSuccess ||
            cudaFuncSetAttribute(mx_gemm_pair_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 kGemmPairSmemGrouped) != cudaSuccess ||
            cudaFuncSetAttribute(mx_gemm_pair_kernel<true, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 kGemmPairSmemGrouped) != cudaSuccess)
            return nullptr;
        d.pair_clusters[0] = max_pair_clusters(mx_gemm_pair_kernel<false>, kGemmPairSmemDense, d.sms);
        d.pair_clusters[1] = max_pair_clusters(mx_gemm_pair_kernel<true>, kGemmPairSmemGrouped, d.sms);
        d.ok = true;
    }
    return &d;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

mx_status check_device(const DeviceInfo** out) {
    const DeviceInfo* d = device_info();
    if (!d) return MX_ERR_CUDA;
    if (d->cc_major != 10) return MX_ERR_UNSUPPORTED;
    *out = d;
    return MX_OK;
}

mx_status launched() { return cudaGetLastError() == cudaSuccess ? MX_OK : MX_ERR_CUDA; }

// cuTensorMapEncodeTiled from the driver, looked up once (no link-time dependency on libcuda).
EncodeTiledFn encode_fn() {
    std::call_once(g_encode_once, [] {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_encode = reinterpret_cast<EncodeTiledFn>(fn);
    });
    return g_encode;
}

// Encoded 2-D tensor maps, cached per host thread. A map is a pure function of its arguments (base
// address, sizes, stride, box, element type, swizzle), so a cached map is never stale; the cache only
// saves the driver call (a few microseconds of host time per map) on repeated calls.
struct TmapKey {
    uintptr_t base;
    uint64_t d0, d1, stride;
    uint32_t b0, b1, kind;
    bool operator==(const TmapKey& o) const {
        return base == o.base && d0 == o.d0 && d1 == o.d1 && stride == o.stride && b0 == o.b0 && b1 == o.b1 &&
               kind == o.kind;
    }
};
struct TmapKeyHash {
    size_t operator()(const TmapKey& k) const {
        uint64_t h = k.base * 0x9E3779B97F4A7C15ull;
        for (uint64_t v : {k.d0, k.d1, k.stride, uint64_t(k.b0) << 32 | k.b1, uint64_t(k.kind)})
            h = (h ^ v) * 0x100000001B3ull;
        return static_cast<size_t>(h ^ (h >> 29));
    }
};
constexpr size_t kTmapCacheMax = 4096;

// kind: 0 = E4M3 operand (uint8, 128-byte swizzle), 1 = scale layout (uint8, no swizzle),
// 2 = BF16 quantizer input (128-byte swizzle).
bool encode_2d(CUtensorMap* map, uint32_t kind, const void* base, uint64_t d0, uint64_t d1, uint64_t stride,
               uint32_t b0, uint32_t b1) {
    static thread_local std::unordered_map<TmapKey, CUtensorMap, TmapKeyHash> cache;
    const TmapKey key{reinterpret_cast<uintptr_t>(base), d0, d1, stride, b0, b1, kind};
    auto it = cache.find(key);
    if (it != cache.end()) {
        *map = it->second;
        return true;
    }
    if (!encode_fn()) return false;
    const cuuint64_t dims[2] = {d0, d1};
    const cuuint64_t strides[1] = {stride};
    const cuuint32_t box[2] = {b0, b1};
    const cuuint32_t estr[2] = {1, 1};
    const CUtensorMapDataType dt = kind == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8;
    const CUtensorMapSwizzle sw = kind == 1 ? CU_TENSOR_MAP_SWIZZLE_NONE : CU_TENSOR_MAP_SWIZZLE_128B;
    if (g_encode(map, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                 CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return false;
    if (cache.size() >= kTmapCacheMax) cache.clear();
    cache.emplace(key, *map);
    return true;
}

// Tensor map of a K-major E4M3 operand [rows, cols_bytes]: boxes of box_rows x box_cols bytes with
// the 128-byte swizzle the UMMA descriptors expect.
bool make_tmap(CUtensorMap* map, const void* base, uint64_t cols_bytes, uint64_t rows, uint32_t box_cols,
               uint32_t box_rows) {
    return encode_2d(map, 0, base, cols_bytes, rows, cols_bytes, box_cols, box_rows);
}

int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

// Checks shared by both GEMMs. Sets *empty when there is nothing to compute (then pointers may be
// null). The output may have any element alignment; 16-byte aligned rows take vector stores.
mx_status gemm_checks(const void* qa, const void* sa, const void* qb, const void* sb, int64_t M, int64_t N,
                      int64_t K, const void* c, int64_t ld_c, mx_out_dtype dt, bool* empty) {
    if (M < 0 || N < 0 || K <= 0 || (dt != MX_OUT_F32 && dt != MX_OUT_BF16)) return MX_ERR_ARG;
    if (K % 32 != 0 || M >= (int64_t(1) << 31) || N >= (int64_t(1) << 31) || K >= (int64_t(1) << 31))
        return MX_ERR_SHAPE;
    if (ld_c < N) return MX_ERR_SHAPE;
    *empty = (M == 0 || N == 0);
    if (*empty) return MX_OK;
    if (!qa || !sa || !qb || !sb || !c) return MX_ERR_ARG;
    const int64_t esz = dt == MX_OUT_BF16 ? 2 : 4;
    if (!aligned16(qa) || !aligned16(sa) || !aligned16(qb) || !aligned16(sb) ||
        (reinterpret_cast<uintptr_t>(c) % esz) != 0)
        return MX_ERR_ALIGN;
    return MX_OK;
}

int vector_store_ok(const void* c, int64_t ld_c, mx_out_dtype dt) {
    const int64_t esz = dt == MX_OUT_BF16 ? 2 : 4;
    return aligned16(c) && (ld_c * esz) % 16 == 0;
}

// Tensor map over a tensor-core scale layout of `blocks` 512-byte blocks, viewed as rows of 256
// bytes: one block is a 2-row box (loaded by the CTA-pair GEMM through TMA so that the peer CTA's
// copies count on the leader's barrier).
bool make_tmap_sf(CUtensorMap* map, const void* base, int64_t blocks) {
    return encode_2d(map, 1, base, 256, static_cast<uint64_t>(2 * blocks), 256, 256, 2);
}

// Launches the CTA-pair GEMM with a cluster dimension of 2.
template <bool GROUPED, int EPI = 0>
mx_status launch_pair(int pairs, const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& tsa,
                      const CUtensorMap& tsb, const GemmArgs& a, mx_stream stream) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * pairs, 1, 1);
    cfg.blockDim = dim3(kGemmThreads, 1, 1);
    cfg.dynamicSmemBytes = GROUPED ? kGemmPairSmemGrouped : kGemmPairSmemDense;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, mx_gemm_pair_kernel<GROUPED, EPI>, ta, tb, tsa, tsb, a) != cudaSuccess) {
        cudaGetLastError();
        return MX_ERR_CUDA;
    }
    return launched();
}

}  // namespace
}  // namespace mx

using namespace mx;

extern "C" {

int64_t mx_swizzled_scale_bytes(int64_t rows, int64_t kblocks) {
    if (rows < 0 || kblocks < 0) return -1;
    return ceil_div(rows, 128) * 128 * (ceil_div(kblocks, 4) * 4);
}

const char* mx_status_string(mx_status s) {
    switch (s) {
        case MX_OK: return "MX_OK";
        case MX_ERR_ARG: return "MX_ERR_ARG: invalid argument";
        case MX_ERR_SHAPE: return "MX_ERR_SHAPE: unsupported shape";
        case MX_ERR_ALIGN: return "MX_ERR_ALIGN: pointer or stride not 16-byte aligned";
        case MX_ERR_CUDA: return "MX_ERR_CUDA: CUDA launch or driver call failed";
        case MX_ERR_UNSUPPORTED: return "MX_ERR_UNSUPPORTED: device is not sm_100";
        case MX_ERR_DEVICE: return "MX_ERR_DEVICE: a kernel reported a device-side error";
    }
    return "unknown mx_status";
}

void mx_set_wait_timeout_ns(uint64_t ns) { g_timeout_ns.store(ns ? ns : kDefaultTimeoutNs); }

mx_status mx_device_error(uint32_t* bits) {
    if (!bits) return MX_ERR_ARG;
    const DeviceInfo* d = nullptr;
    if (mx_status st = check_device(&d)) return st;
    uint32_t v = 0;
    if (cudaDeviceSynchronize() != cudaSuccess) return MX_ERR_CUDA;
    if (cudaMemcpy(&v, d->status, sizeof v, cudaMemcpyDeviceToHost) != cudaSuccess) return MX_ERR_CUDA;
    const uint32_t zero = 0;
    if (cudaMemcpy(d->status, &zero, sizeof zero, cudaMemcpyHostToDevice) != cudaSuccess) return MX_ERR_CUDA;
    *bits = v;
    return v ? MX_ERR_DEVICE : MX_OK;
}

mx_status mx_diag_expired_wait(mx_stream stream) {
    const DeviceInfo* d = nullptr;
    if (mx_status st = check_device(&d)) return st;
    expired_wait_kernel<<<1, 32, 0, stream>>>(d->status, g_timeout_ns.load());
    return launched();
}

}  // extern "C"

namespace mx {
namespace {

// Validates one tensor of a quantize call; *empty is set when it has no elements.
mx_status check_quant_tensor(const mx_quant_tensor& t, bool row, bool col, bool* empty) {
    if (t.M < 0 || t.K < 0) return MX_ERR_ARG;
    if (t.K % 32 != 0 || (col && t.M % 32 != 0)) return MX_ERR_SHAPE;
    if (t.M >= (int64_t(1) << 31) || t.K >= (int64_t(1) << 31)) return MX_ERR_SHAPE;
    *empty = (t.M == 0 || t.K == 0);
    if (*empty) return MX_OK;   // empty tensors may carry null pointers
    if (!t.x || (row && (!t.q_row || !t.s_row)) || (col && (!t.q_col || !t.s_col))) return MX_ERR_ARG;
    if (t.ld_x < t.K) return MX_ERR_SHAPE;
    if (!aligned16(t.x) || t.ld_x % 8 != 0) return MX_ERR_ALIGN;
    if (row && (!aligned16(t.q_row) || !aligned16(t.s_row))) return MX_ERR_ALIGN;
    if (col && (!aligned16(t.q_col) || !aligned16(t.s_col))) return MX_ERR_ALIGN;
    return MX_OK;
}

template <int NT>
void add_quant_tensor(QuantArgs<NT>& a, const mx_quant_tensor& t) {
    QTensor& q = a.t[a.n++];
    q.x = static_cast<const uint16_t*>(t.x);
    q.q_row = t.q_row;
    q.s_row = t.s_row;
    q.q_col = t.q_col;
    q.s_col = t.s_col;
    q.M = t.M;
    q.K = t.K;
    q.ldx = t.ld_x;
    q.tiles_m = static_cast<int32_t>(ceil_div(t.M, kQTile));
    q.tiles_k = static_cast<int32_t>(ceil_div(t.K, kQTile));
    q.vec32 = (reinterpret_cast<uintptr_t>(t.x) % 32 == 0) && (t.ld_x % 16 == 0) &&
              (reinterpret_cast<uintptr_t>(t.q_row) % 32 == 0);
    q.col_vec32 = reinterpret_cast<uintptr_t>(t.q_col) % 32 == 0;
    q.tile_start = a.total_tiles;
    a.total_tiles += int64_t(q.tiles_m) * q.tiles_k;
}

template <int NT>
mx_status launch_quant(const QuantArgs<NT>& a, bool row, bool col, const DeviceInfo* d, mx_stream stream) {
    if (a.total_tiles == 0) return MX_OK;
    const int which = (row ? 1 : 0) | (col ? 2 : 0);
    const int64_t grid = std::min<int64_t>(a.total_tiles, int64_t(d->sms) * d->quant_blocks_per_sm[which]);
    const int v = g_quant_variant.load();
    if (col)     // row + col (columnwise only takes the TMA-staged kernel)
        quantize_rowcol_kernel<true, NT><<<grid, kQThreads, 0, stream>>>(a);
    else if (v == 2 || (v == 0 && a.total_tiles >= kSplitTilesPerCta * grid))
        quantize_rowwise_kernel<NT, true><<<grid, kQThreads, 0, stream>>>(a);
    else
        quantize_rowwise_kernel<NT, false><<<grid, kQThreads, 0, stream>>>(a);
    return launched();
}

// Tensor map of a BF16 input [M, K] (row stride ld_x elements) in 64-column x 128-row boxes with the
// 128-byte swizzle the TMA-staged quantizer reads; out-of-range elements arrive as zeros.
bool make_tmap_bf16(CUtensorMap* map, const void* base, int64_t M, int64_t K, int64_t ld_x) {
    return encode_2d(map, 2, base, static_cast<uint64_t>(K), static_cast<uint64_t>(M), static_cast<uint64_t>(ld_x) * 2,
                     64, 128);
}

template <int NT>
bool add_qt_tensor(QuantTmaArgs<NT>& a, const mx_quant_tensor& t) {
    const int i = a.n;
    if (!make_tmap_bf16(&a.map[i], t.x, t.M, t.K, t.ld_x)) return false;
    QtTensor& q = a.t[i];
    q.q_row = t.q_row;
    q.s_row = t.s_row;
    q.q_col = t.q_col;
    q.s_col = t.s_col;
    q.M = static_cast<int32_t>(t.M);
    q.K = static_cast<int32_t>(t.K);
    q.tiles_m = static_cast<int32_t>(ceil_div(t.M, kQTile));
    q.tiles_k = static_cast<int32_t>(ceil_div(t.K, kQTile));
    q.vec32 = reinterpret_cast<uintptr_t>(t.q_row) % 32 == 0;
    q.col_vec32 = reinterpret_cast<uintptr_t>(t.q_col) % 32 == 0;
    q.tile_start = a.total_tiles;
    a.total_tiles += int64_t(q.tiles_m) * q.tiles_k;
    ++a.n;
    return true;
}

template <int NT>
mx_status launch_qt(const QuantTmaArgs<NT>& a, bool row, bool col, const DeviceInfo* d, mx_stream stream) {
    if (a.total_tiles == 0) return MX_OK;
    const int which = (row ? 1 : 0) | (col ? 2 : 0);
    const int64_t grid = std::min<int64_t>(a.total_tiles, int64_t(d->sms) * d->qt_blocks_per_sm[which]);
    if (row && col)
        quantize_tma_kernel<true, true, NT><<<grid, kQThreads, kQtSmemBytes, stream>>>(a);
    else if (row)
        quantize_tma_kernel<true, false, NT><<<grid, kQThreads, kQtSmemBytes, stream>>>(a);
    else
        quantize_tma_kernel<false, true, NT><<<grid, kQThreads, kQtSmemBytes, stream>>>(a);
    return launched();
}

template <int NP>
void add_pair(CmpArgs<NP>& g, const uint8_t* a, const uint8_t* b, int64_t nbytes) {
    CmpPair& p = g.p[g.n++];
    p.a = a;
    p.b = b;
    p.nbytes = nbytes;
    p.vec = aligned16(a) && aligned16(b);
    p.unit_start = g.total_units;
    g.total_units += ceil_div(nbytes, kGeUnitBytes);
}

template <int NP>
mx_status launch_compare(const CmpArgs<NP>& g, const DeviceInfo* d, mx_stream stream) {
    grid_equal_reset_kernel<<<static_cast<int>(ceil_div(g.n, 256)), 256, 0, stream>>>(g.counts, g.firsts, g.n);
    if (mx_status st = launched()) return st;
    if (g.total_units == 0) return MX_OK;
    const int64_t grid = std::min<int64_t>(g.total_units, int64_t(d->sms) * d->ge_blocks_per_sm);
    grid_equal_kernel<NP><<<grid, kGeThreads, 0, stream>>>(g);
    return launched();
}

}  // namespace
}  // namespace mx

extern "C" {

mx_status mx_quantize(const void* x, int64_t M, int64_t K, int64_t ld_x, int flags, uint8_t* q_row,
                      uint8_t* s_row, uint8_t* q_col, uint8_t* s_col, mx_stream stream) {
    const bool row = flags & MX_ROWWISE, col = flags & MX_COLWISE, swz = flags & MX_SWIZZLE;
    if (flags & ~(MX_ROWWISE | MX_COLWISE | MX_SWIZZLE)) return MX_ERR_ARG;
    if (!row && !col) return MX_ERR_ARG;
    const mx_quant_tensor t{x, M, K, ld_x, q_row, s_row, q_col, s_col};
    bool empty = false;
    if (mx_status st = check_quant_tensor(t, row, col, &empty)) return st;
    if (empty) return MX_OK;
    const DeviceInfo* d = nullptr;
    if (mx_status st = check_device(&d)) return st;
    if (use_tma_quantizer(row, col)) {
        QuantTmaArgs<1> a;
        a.n = 0;
        a.swz = swz;
        a.total_tiles = 0;
        a.err = d->status;
        a.timeout_ns = g_timeout_ns.load();
        if (!add_qt_tensor(a, t)) return MX_ERR_CUDA;
        return launch_qt(a, row, col, d, stream);
    }
    QuantArgs<1> a;
    a.n = 0;
    a.swz = swz;
    a.total_tiles = 0;
    add_quant_tensor(a, t);
    return launch_quant(a, row, col, d, stream);
}

mx_status mx_quantize_multi(const mx_quant_tensor* tensors, int64_t n, int flags, mx_stream stream) {
    const bool row = flags & MX_ROWWISE, col = flags & MX_COLWISE, swz = flags & MX_SWIZZLE;
    if (flags & ~(MX_ROWWISE | MX_COLWISE | MX_SWIZZLE)) return MX_ERR_ARG;
    if (!row && !col) return MX_ERR_ARG;
    if (n < 0 || (n > 0 && !tensors)) return MX_ERR_ARG;
    for (int64_t i = 0; i < n; ++i) {
        bool empty = false;
        if (mx_status st = check_quant_tensor(tensors[i], row, col, &empty)) return st;
    }
    if (n == 0) return MX_OK;
    const DeviceInfo* d = nullptr;
    if (mx_status st = check_device(&d)) return st;
    if (use_tma_quantizer(row, col)) {
        static thread_local QuantTmaArgs<kQtMaxTensors> a;   // ~30 KB: kept off the stack
        for (int64_t i0 = 0; i0 < n; i0 += kQtMaxTensors) {
            a.n = 0;
            a.swz = swz;
            a.total_tiles = 0;
            a.err = d->status;
            a.timeout_ns = g_timeout_ns.load();
            for (int64_t i = i0; i < std::min<int64_t>(n, i0 + kQtMaxTensors); ++i) {
                const mx_quant_tensor& t = tensors[i];
                if (t.M > 0 && t.K > 0 && !add_qt_tensor(a, t)) return MX_ERR_CUDA;
            }
            if (a.n == 0) continue;
            if (mx_status st = launch_qt(a, row, col, d, stream)) return st;
        }
        return MX_OK;
    }
    static thread_local QuantArgs<kQMaxTensors> a;   // ~14 KB: kept off the stack
    for (int64_t i0 = 0; i0 < n; i0 += kQMaxTensors) {
        a.n = 0;
        a.swz = swz;
        a.total_tiles = 0;
        for (int64_t i = i0; i < std::min<int64_t>(n, i0 + kQMaxTensors); ++i) {
            const mx_quant_tensor& t = tensors[i];
            if (t.M > 0 && t.K > 0) add_quant_tensor(a, t);
        }
        if (a.n == 0) continue;
        if (mx_status st = launch_quant(a, row, col, d, stream)) return st;
    }
    return MX_OK;
}

mx_status mx_swizzle_scales(const uint8_t* s, int64_t rows, int64_t kblocks, const int64_t* group_rows_host,
                            int64_t groups, uint8_t* s_swz, mx_stream stream) {
    if (rows < 0 || kblocks < 0) return MX_ERR_ARG;
    if (group_rows_host && groups < 1) return MX_ERR_ARG;
    if (group_rows_host) {
        int64_t total = 0;
        for (int64_t g = 0; g < groups; ++g) {
            if (group_rows_host[g] < 0) return MX_ERR_ARG;
            total += group_rows_host[g];
        }
        if (total != rows) return MX_ERR_SHAPE;
    }
    if (rows == 0 || kblocks == 0) return MX_OK;   // empty: pointers may be NULL
    if (!s || !s_swz) return MX_ERR_ARG;
    if (!aligned16(s_swz)) return MX_ERR_ALIGN;
    const DeviceInfo* d = nullptr;
    if (mx_status st = check_device(&d)) return st;

    const int64_t one = rows;
    const int64_t* gr = group_rows_host ? group_rows_host : &one;
    const int64_t ng = group_rows_host ? groups : 1;
    const int64_t ctiles = ceil_div(kblocks, 4);
    const bool quad = kblocks % 16 == 0 && aligned16(s);
    int64_t src_row = 0, out_block = 0;
    for (int64_t g0 = 0; g0 < ng; g0 += kSwzMaxGroups) {
        SwizzleArgs a;
        a.s = s;
        a.kblocks = kblocks;
        a.ctiles = ctiles;
        a.word_loads = kblocks % 4 == 0 && (reinterpret_cast<uintptr_t>(s) & 3u) == 0;
        a.ngroups = static_cast<int>(std::min<int64_t>(kSwzMaxGroups, ng - g0));
        a.out = s_swz + out_block * 512;
        int64_t local_block = 0;
        for (int i = 0; i < a.ngroups; ++i) {
            a.src_row[i] = src_row;
            a.rows[i] = gr[g0 + i];
            a.block_start[i] = local_block;
            local_block += ceil_div(gr[g0 + i], 128) * ctiles;
            src_row += gr[g0 + i];
        }
        a.block_start[a.ngroups] = local_block;
        if (local_block > 0) {
            const int64_t warps = quad ? local_block / 4 : local_block;
            const int64_t grid = std::min<int64_t>(ceil_div(warps * 32, 256), int64_t(d->sms) * 16);
            if (quad)
                swizzle_kernel<true><<<grid, 256, 0, stream>>>(a);
            else
                swizzle_kernel<false><<<grid, 256, 0, stream>>>(a);
            if (mx_status st = launched()) return st;
        }
        out_block += local_block;
    }
    return MX_OK;
}

mx_status mx_grid_equal(const uint8_t* a, const uint8_t* b, int64_t nbytes, unsigned long long* mismatches_dev,
                        long long* first_index_dev, mx_stream stream) {
    if (!mismatches_dev || !first_index_dev || nbytes < 0 || (nbytes > 0 && (!a || !b))) return MX_ERR_ARG;
    const DeviceInfo* d = nullptr;
    if (mx_status st = check_device(&d)) return st;
    CmpArgs<1> g;
    g.n = 0;
    g.total_units = 0;
    g.counts = mismatches_dev;
    g.firsts = first_index_dev;
    add_pair(g, a, b, nbytes);
    return launch_compare(g, d, stream);
}

mx_status mx_grid_equal_multi(const mx_compare_pair* pairs, int64_t n, unsigned long long* mismatches_dev,
                              long long* first_index_dev, mx_stream stream) {
    if (n < 0 || (n > 0 && (!pairs || !mismatches_dev || !first_index_dev))) return MX_ERR_ARG;
    for (int64_t i = 0; i < n; ++i)
        if (pairs[i].nbytes < 0 || (pairs[i].nbytes > 0 && (!pairs[i].a || !pairs[i].b))) return MX_ERR_ARG;
    if (n == 0) return MX_OK;
    const DeviceInfo* d = nullptr;
    if (mx_status st = check_device(&d)) return st;
    static thread_local CmpArgs<kGeMaxPairs> g;      // ~20 KB: kept off the stack
    for (int64_t i0 = 0; i0 < n; i0 += kGeMaxPairs) {
        g.n = 0;
        g.total_units = 0;
        g.counts = mismatches_dev + i0;
        g.firsts = first_index_dev + i0;
        for (int64_t i = i0; i < std::min<int64_t>(n, i0 + kGeMaxPairs); ++i)
            add_pair(g, pairs[i].a, pairs[i].b, pairs[i].nbytes);
        if (mx_status st = launch_compare(g, d, stream)) return st;
    }
    return MX_OK;
}

mx_status mx_quantize_compare_multi(const mx_quant_tensor* tensors, const mx_grid_ref* refs, int64_t n,
                                    unsigned long long* mismatches_dev, long long* first_index_dev,
                                    mx_stream stream) {
    if (n < 0 || n > (int64_t(1) << 30) || (n > 0 && (!tensors || !refs || !mismatches_dev || !first_index_dev)))
        return MX_ERR_ARG;
    for (int64_t i = 0; i < n; ++i) {
        bool empty = false;
        if (mx_status st = check_quant_tensor(tensors[i], true, false, &empty)) return st;
        if (empty) continue;
        if (!refs[i].q || !refs[i].s) return MX_ERR_ARG;
        if (!aligned16(refs[i].q) || !aligned16(refs[i].s)) return MX_ERR_ALIGN;
    }
    if (n == 0) return MX_OK;
    const DeviceInfo* d = nullptr;
    if (mx_status st = check_device(&d)) return st;
    const int64_t slots = 2 * n;
    grid_equal_reset_kernel<<<static_cast<int>(std::min<int64_t>(ceil_div(slots, 256), 1024)), 256, 0, stream>>>(
        mismatches_dev, first_index_dev, static_cast<int>(slots));
    if (mx_status st = launched()) return st;
    static thread_local QuantArgs<kQMaxTensors> a;   // ~20 KB: kept off the stack
    for (int64_t i0 = 0; i0 < n; i0 += kQMaxTensors) {
        a.n = 0;
        a.swz = 1;
        a.total_tiles = 0;
        a.cmp_counts = mismatches_dev;
        a.cmp_firsts = first_index_dev;
        for (int64_t i = i0; i < std::min<int64_t>(n, i0 + kQMaxTensors); ++i) {
            const mx_quant_tensor& t = tensors[i];
            if (t.M == 0 || t.K == 0) continue;
            add_quant_tensor(a, t);
            QTensor& q = a.t[a.n - 1];
            q.ref_q = refs[i].q;
            q.ref_s = refs[i].s;
            q.res = static_cast<int32_t>(i);
            q.ref_vec32 = reinterpret_cast<uintptr_t>(refs[i].q) % 32 == 0;
        }
        if (a.n == 0) continue;
        const int64_t grid = std::min<int64_t>(a.total_tiles, int64_t(d->sms) * d->quant_blocks_per_sm[1]);
        if (a.total_tiles >= kSplitTilesPerCta * grid)
            quantize_rowwise_kernel<kQMaxTensors, true, true><<<grid, kQThreads, 0, stream>>>(a);
        else
            quantize_rowwise_kernel<kQMaxTensors, false, true><<<grid, kQThreads, 0, stream>>>(a);
        if (mx_status st = launched()) return st;
    }
    return MX_OK;
}

mx_status mx_gemm(const uint8_t* qa, const uint8_t* sa_swz, const uint8_t* qb, const uint8_t* sb_swz, int64_t M,
                  int64_t N, int64_t K, void* c, int64_t ld_c, mx_out_dtype out_dtype, mx_stream stream) {
    bool empty = false;
    if (mx_status st = gemm_checks(qa, sa_swz, qb, sb_swz, M, N, K, c, ld_c, out_dtype, &empty)) return st;
    if (empty) return MX_OK;
    const DeviceInfo* d = nullptr;
    if (mx_status st = check_device(&d)) return st;
    const bool pair = g_gemm_variant.load() == 0;
    GemmArgs a{};
    a.sfa = sa_swz;
    a.sfb = sb_swz;
    a.c = c;
    a.ldc = ld_c;
    a.M = static_cast<int>(M);
    a.N = static_cast<int>(N);
    a.K = static_cast<int>(K);
    a.nkb = static_cast<int>(ceil_div(K, kBK));
    a.tiles_m = static_cast<int>(ceil_div(M, pair ? 2 * kBM : kBM));
    a.tiles_n = static_cast<int>(ceil_div(N, kBN));
    a.sfa_tiles = static_cast<int>(ceil_div(M, 128));
    a.out_bf16 = out_dtype == MX_OUT_BF16;
    a.vec_store = vector_store_ok(c, ld_c, out_dtype);
    a.G = 1;
    a.n_fast = M > N;      // A is the larger operand: walk N fastest so B (the smaller) stays in L2
    a.n_rowtiles = static_cast<int>(ceil_div(N, 128));
    a.row_offsets = nullptr;
    a.err = d->status;
    a.timeout_ns = g_timeout_ns.load();
    CUtensorMap ta, tb;
    const int64_t tiles = int64_t(a.tiles_m) * a.tiles_n;
    if (pair) {
        CUtensorMap tsa, tsb;
        if (!make_tmap(&ta, qa, K, M, kBK, kBM) || !make_tmap(&tb, qb, K, N, kBK, kBN / 2) ||
            !make_tmap_sf(&tsa, sa_swz, int64_t(a.sfa_tiles) * a.nkb) ||
            !make_tmap_sf(&tsb, sb_swz, int64_t(a.n_rowtiles) * a.nkb))
            return MX_ERR_CUDA;
        const int pairs = static_cast<int>(std::min<int64_t>(tiles, d->pair_clusters[0]));
        return launch_pair<false>(pairs, ta, tb, tsa, tsb, a, stream);
    }
    if (!make_tmap(&ta, qa, K, M, kBK, kBM) || !make_tmap(&tb, qb, K, N, kBK, kBN)) return MX_ERR_CUDA;
    const int grid = static_cast<int>(std::min<int64_t>(tiles, d->sms));
    mx_gemm_kernel<false><<<grid, kGemmThreads, kGemmSmemDense, stream>>>(ta, tb, a);
    return launched();
}

mx_status mx_grouped_gemm(const uint8_t* qa, const uint8_t* sa_swz, const uint8_t* qb, const uint8_t* sb_swz,
                          const int32_t* row_offsets_dev, int64_t G, int64_t total_rows, int64_t N, int64_t K,
                          void* c, int64_t ld_c, mx_out_dtype out_dtype, mx_stream stream) {
    if (!row_offsets_dev || G < 1) return MX_ERR_ARG;
    if (G > kMaxGroups) return MX_ERR_SHAPE;
    if (reinterpret_cast<uintptr_t>(row_offsets_dev) & 3u) return MX_ERR_ALIGN;
    bool empty = false;
    if (mx_status st = gemm_checks(qa, sa_swz, qb, sb_swz, total_rows, N, K, c, ld_c, out_dtype, &empty))
        return st;
    if (G * N >= (int64_t(1) << 31)) return MX_ERR_SHAPE;
    if (empty) return MX_OK;
    const DeviceInfo* d = nullptr;
    if (mx_status st = check_device(&d)) return st;
    const bool pair = g_gemm_variant.load() == 0;
    GemmArgs a{};
    a.sfa = sa_swz;
    a.sfb = sb_swz;
    a.c = c;
    a.ldc = ld_c;
    a.M = static_cast<int>(total_rows);
    a.N = static_cast<int>(N);
    a.K = static_cast<int>(K);
    a.nkb = static_cast<int>(ceil_div(K, kBK));
    a.tiles_m = 0;
    a.tiles_n = static_cast<int>(ceil_div(N, kBN));
    a.sfa_tiles = 0;
    a.out_bf16 = out_dtype == MX_OUT_BF16;
    a.vec_store = vector_store_ok(c, ld_c, out_dtype);
    a.G = static_cast<int>(G);
    a.n_rowtiles = static_cast<int>(ceil_div(N, 128));
    a.row_offsets = row_offsets_dev;
    a.err = d->status;
    a.timeout_ns = g_timeout_ns.load();
    CUtensorMap ta, tb;
    if (pair) {
        // Upper bounds: every group adds at most one partial 256-row tile, one partial 128-row scale tile.
        const int64_t max_tiles = (ceil_div(total_rows, 2 * kBM) + G) * a.tiles_n;
        CUtensorMap tsa, tsb;
        if (!make_tmap(&ta, qa, K, total_rows, kBK, kBM) || !make_tmap(&tb, qb, K, G * N, kBK, kBN / 2) ||
            !make_tmap_sf(&tsa, sa_swz, (ceil_div(total_rows, 128) + G) * a.nkb) ||
            !make_tmap_sf(&tsb, sb_swz, G * a.n_rowtiles * a.nkb))
            return MX_ERR_CUDA;
        const int pairs = static_cast<int>(std::min<int64_t>(max_tiles, d->pair_clusters[1]));
        return launch_pair<true>(pairs, ta, tb, tsa, tsb, a, stream);
    }
    if (!make_tmap(&ta, qa, K, total_rows, kBK, kBM) || !make_tmap(&tb, qb, K, G * N, kBK, kBN))
        return MX_ERR_CUDA;
    // Upper bound on tiles: every group adds at most one partial 128-row tile.
    const int64_t max_tiles = (ceil_div(total_rows, kBM) + G) * a.tiles_n;
    const int grid = static_cast<int>(std::min<int64_t>(max_tiles, d->sms));
    mx_gemm_kernel<true><<<grid, kGemmThreads, kGemmSmemGrouped, stream>>>(ta, tb, a);
    return launched();
}

mx_status mx_grouped_gemm_swiglu_quant(const uint8_t* qa, const uint8_t* sa_swz, const uint8_t* qb,
                                       const uint8_t* sb_swz, const int32_t* row_offsets_dev, int64_t G,
                                       int64_t total_rows, int64_t n_inter, int64_t K, uint8_t* h_q,
                                       uint8_t* h_s_swz, mx_stream stream) {
    if (!row_offsets_dev || G < 1 || n_inter <= 0) return MX_ERR_ARG;
    if (G > kMaxGroups || n_inter % 128 != 0) return MX_ERR_SHAPE;
    if (reinterpret_cast<uintptr_t>(row_offsets_dev) & 3u) return MX_ERR_ALIGN;
    const int64_t N = 2 * n_inter;
    bool empty = false;
    // Operand and shape checks of the GEMM (its C argument stands in for h_q here; h_q and h_s_swz
    // get their own 16-byte alignment check below).
    if (mx_status st = gemm_checks(qa, sa_swz, qb, sb_swz, total_rows, N, K, h_q, N, MX_OUT_BF16, &empty))
        return st;
    if (G * N >= (int64_t(1) << 31)) return MX_ERR_SHAPE;
    if (empty) return MX_OK;
    if (!h_s_swz) return MX_ERR_ARG;
    if (!aligned16(h_q) || !aligned16(h_s_swz)) return MX_ERR_ALIGN;
    const DeviceInfo* d = nullptr;
    if (mx_status st = check_device(&d)) return st;
    GemmArgs a{};
    a.sfa = sa_swz;
    a.sfb = sb_swz;
    a.M = static_cast<int>(total_rows);
    a.N = static_cast<int>(N);
    a.K = static_cast<int>(K);
    a.nkb = static_cast<int>(ceil_div(K, kBK));
    a.tiles_n = static_cast<int>(N / kBN);
    a.G = static_cast<int>(G);
    a.n_rowtiles = static_cast<int>(N / 128);
    a.row_offsets = row_offsets_dev;
    a.err = d->status;
    a.timeout_ns = g_timeout_ns.load();
    a.hq = h_q;
    a.hs = h_s_swz;
    a.n_inter = static_cast<int>(n_inter);
    a.hs_ctiles = static_cast<int>(n_inter / 128);
    const int64_t max_tiles = (ceil_div(total_rows, 2 * kBM) + G) * a.tiles_n;
    CUtensorMap ta, tb, tsa, tsb;
    if (!make_tmap(&ta, qa, K, total_rows, kBK, kBM) || !make_tmap(&tb, qb, K, G * N, kBK, kBN / 2) ||
        !make_tmap_sf(&tsa, sa_swz, (ceil_div(total_rows, 128) + G) * a.nkb) ||
        !make_tmap_sf(&tsb, sb_swz, G * a.n_rowtiles * a.nkb))
        return MX_ERR_CUDA;
    const int pairs = static_cast<int>(std::min<int64_t>(max_tiles, d->pair_clusters[1]));
    return launch_pair<true, 1>(pairs, ta, tb, tsa, tsb, a, stream);
}

mx_status mx_quantize_block128(const void* x, int64_t M, int64_t K, int64_t ld_x, int pow2_scales, uint8_t* q,
                               float* scales, mx_stream stream) {
    if (M < 0 || K < 0) return MX_ERR_ARG;
    if (K % 32 != 0 || M >= (int64_t(1) << 31) || K >= (int64_t(1) << 31)) return MX_ERR_SHAPE;
    if (M == 0 || K == 0) return MX_OK;                // empty: pointers may be NULL
    if (!x || !q || !scales) return MX_ERR_ARG;
    if (ld_x < K) return MX_ERR_SHAPE;
    if (!aligned16(x) || ld_x % 8 != 0 || !aligned16(q) || (reinterpret_cast<uintptr_t>(scales) & 3u))
        return MX_ERR_ALIGN;
    const DeviceInfo* d = nullptr;
    if (mx_status st = check_device(&d)) return st;
    Block128Args a;
    a.x = static_cast<const uint16_t*>(x);
    a.q = q;
    a.scales = scales;
    a.M = M;
    a.K = K;
    a.ldx = ld_x;
    a.tiles_m = static_cast<int>(ceil_div(M, kQTile));
    a.tiles_k = static_cast<int>(ceil_div(K, kQTile));
    a.pow2 = pow2_scales != 0;
    a.vec32 = (reinterpret_cast<uintptr_t>(x) % 32 == 0) && (ld_x % 16 == 0) &&
              (reinterpret_cast<uintptr_t>(q) % 32 == 0);
    const int64_t tiles = int64_t(a.tiles_m) * a.tiles_k;
    if (a.pow2)
        quantize_block128_kernel<true><<<std::min<int64_t>(tiles, int64_t(d->sms) * 2), kQThreads, 0, stream>>>(a);
    else
        quantize_block128_kernel<false><<<std::min<int64_t>(tiles, int64_t(d->sms) * 4), kQThreads, 0, stream>>>(a);
    return launched();
}

void mx_set_gemm_variant(int variant) { g_gemm_variant.store(variant == 1 ? 1 : 0); }

void mx_set_quantize_variant(int variant) { g_quant_variant.store(variant == 1 || variant == 2 ? variant : 0); }

}  // extern "C"
