// libmla_b200.so: the C ABI of include/mla.h. This is the library's single translation
// unit; the kernels live in the headers it includes.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <vector>

#include "mla.h"

#include "append.cuh"
#include "append_fp8.cuh"
#include "combine.cuh"
#include "common.cuh"
#include "decode_simt.cuh"
#include "decode_pair.cuh"
#include "decode_solo.cuh"
#include "metadata.cuh"
#include "rank_combine.cuh"
#include "sched.cuh"

// Split-partial scratch of mla_decode_fwd_noalloc: a fixed array inside the library in
// place of a caller-provided workspace. One copy exists per device; every call of that
// entry point on the device shares it (see include/mla.h for the rules that follow).
static __device__ __align__(256) unsigned char g_noalloc_scratch[MLA_NOALLOC_SCRATCH_BYTES];

namespace {

using namespace mla;

constexpr size_t kWsHeader = 256;
constexpr size_t kAlign = 256;

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

bool shape_ok(int batch, int h_q, int s_q) {
    return batch >= 1 && batch <= MLA_MAX_BATCH && h_q >= 1 && h_q <= MLA_MAX_H_Q &&
           s_q >= 1 && s_q <= MLA_MAX_S_Q && h_q * s_q <= MLA_MAX_ROWS;
}

// Up to kSoloMaxRows query rows per sequence the 1-CTA kernel (decode_solo.cuh) runs;
// above it the 2-CTA kernel (decode_pair.cuh) splits 128-row tiles over two SMs.
bool use_solo(int h_q, int s_q) { return h_q * s_q <= kSoloMaxRows; }

// Query rows per sequence the FP8-cache decode takes: the 1-CTA kernel's (each page is
// widened in its own stage, so every 1-CTA layout carries it).
constexpr int kFp8MaxRows = kSoloMaxRows;

// Work units a schedule for num_sms SMs may use, before the device cap: one per SM for
// the 1-CTA kernel, one per SM pair for the 2-CTA kernel.
int units_bound(int num_sms, int h_q, int s_q) {
    const int u = use_solo(h_q, s_q) ? num_sms : num_sms / 2;
    return u < 1 ? 1 : u;
}

size_t max_chunks_for(int batch, int h_q, int s_q, int num_sms) {
    return (size_t)batch * num_tiles(h_q, s_q) + (size_t)units_bound(num_sms, h_q, s_q);
}


// Per partial slot: 128 rows' lse and outputs (fp32), and the combine's counters of one
// work sequence (there are never more work sequences than slots).
constexpr size_t kChunkBytes = (size_t)kTileRows * 4 + (size_t)kTileRows * kHeadDimV * 4 +
                               (size_t)kCombineCounters * 4;

// Partial-slot capacity of a workspace and the byte offsets of its output partials and
// combine counters.
size_t ws_capacity(size_t bytes) {
    if (bytes < kWsHeader + 2 * kAlign) return 0;
    return (bytes - kWsHeader - 2 * kAlign) / kChunkBytes;
}

size_t ws_o_offset(size_t cap) { return align_up(kWsHeader + cap * kTileRows * 4, kAlign); }

// The combine counters start right after the output partials (combine_counters()).
size_t ws_cnt_offset(size_t cap) { return ws_o_offset(cap) + cap * kTileRows * kHeadDimV * 4; }

// Workspace bytes that hold `cap` partial slots.
size_t workspace_bytes_for(size_t cap) {
    return ws_cnt_offset(cap) + cap * kCombineCounters * 4 + kAlign;
}

// Opt the split kernel into its shared-memory footprint (once per device).
bool prepare_split_kernel(int dev) {
    static std::mutex mu;
    static std::vector<char> done;
    std::lock_guard<std::mutex> lock(mu);
    if ((int)done.size() <= dev) done.resize(dev + 1, 0);
    if (done[dev]) return true;
    if (cudaFuncSetAttribute(pair::decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)pair::kSmemAlloc) != cudaSuccess)
        return false;
    cudaFuncAttributes attr;
    if (cudaFuncGetAttributes(&attr, pair::decode_kernel) != cudaSuccess) return false;
    if (attr.maxThreadsPerBlock < pair::kThreads) return false;
    done[dev] = 1;
    return true;
}

// Allow the scheduler kernel kMetaSmemMax of dynamic shared memory (once per device).
bool prepare_metadata_kernel() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return false;
    static std::mutex mu;
    static std::vector<char> done;
    std::lock_guard<std::mutex> lock(mu);
    if ((int)done.size() <= dev) done.resize(dev + 1, 0);
    if (done[dev]) return done[dev] > 0;
    const bool ok = cudaFuncSetAttribute(metadata_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kMetaSmemMax) == cudaSuccess;
    if (!ok) cudaGetLastError();
    done[dev] = ok ? 1 : -1;
    return ok;
}

// 2-CTA clusters of the split kernel that can be co-resident on a device (cached per
// device); a schedule never uses more units than this, so every unit runs in one wave.
int device_pairs(int dev) {
    static std::mutex mu;
    static std::vector<int> cache;
    {
        std::lock_guard<std::mutex> lock(mu);
        if ((int)cache.size() > dev && cache[dev] > 0) return cache[dev];
    }
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return -1;
    int pairs = sms / 2 < 1 ? 1 : sms / 2;
    if (prepare_split_kernel(dev)) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(2 * pairs);
        cfg.blockDim = dim3(pair::kThreads);
        cfg.dynamicSmemBytes = pair::kSmemAlloc;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int clusters = 0;
        if (cudaOccupancyMaxActiveClusters(&clusters, pair::decode_kernel, &cfg) == cudaSuccess &&
            clusters > 0 && clusters < pairs)
            pairs = clusters;
        cudaGetLastError();
    }
    std::lock_guard<std::mutex> lock(mu);
    if ((int)cache.size() <= dev) cache.resize(dev + 1, 0);
    cache[dev] = pairs;
    return pairs;
}

template <class C>
bool prepare_solo_kernel(int dev) {
    static std::mutex mu;
    static std::vector<char> done;
    std::lock_guard<std::mutex> lock(mu);
    if ((int)done.size() <= dev) done.resize(dev + 1, 0);
    if (done[dev]) return true;
    if (cudaFuncSetAttribute(solo::decode_kernel<C>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)C::kSmemAlloc) != cudaSuccess)
        return false;
    done[dev] = 1;
    return true;
}

// CTAs of the 1-CTA kernel that can be co-resident on a device (cached per device): one
// per SM, as its shared memory and TMEM allow no second. A schedule never uses more
// units than this, so every unit runs in one wave.
int device_solo_ctas(int dev) {
    static std::mutex mu;
    static std::vector<int> cache;
    {
        std::lock_guard<std::mutex> lock(mu);
        if ((int)cache.size() > dev && cache[dev] > 0) return cache[dev];
    }
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return -1;
    int ctas = sms < 1 ? 1 : sms;
    if (prepare_solo_kernel<solo::Cfg<64>>(dev)) {
        int per_sm = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, solo::decode_kernel<solo::Cfg<64>>,
                                                          solo::Cfg<64>::kBlockThreads,
                                                          solo::Cfg<64>::kSmemAlloc) == cudaSuccess &&
            per_sm >= 1 && per_sm * sms < ctas)
            ctas = per_sm * sms;
        cudaGetLastError();
    }
    std::lock_guard<std::mutex> lock(mu);
    if ((int)cache.size() <= dev) cache.resize(dev + 1, 0);
    cache[dev] = ctas;
    return ctas;
}

// Units of every schedule the current device can run for these shapes.
int device_units(int dev, int h_q, int s_q) {
    return use_solo(h_q, s_q) ? device_solo_ctas(dev) : device_pairs(dev);
}

// cuTensorMapEncodeTiled from the driver, found at run time so the library does not
// link libcuda (it must load on machines without a GPU driver).
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_tiled_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    });
    return fn;
}

// 3-D view of the page pool for the split kernel: {64 elements, num_blocks * 64 rows
// (stride 1152 bytes), 9 chunks of 128 bytes (stride 128 bytes)}, 128-byte swizzle, box
// {64, 64, box_chunks}: a box lands as box_chunks consecutive 64-row x 128-byte tiles.
bool make_page_map(CUtensorMap* map, const void* kcache, int num_blocks, int box_chunks) {
    EncodeTiledFn fn = encode_tiled_fn();
    if (!fn) return false;
    const cuuint64_t dims[3] = {64, (cuuint64_t)num_blocks * kBlock, (cuuint64_t)(kHeadDim / 64)};
    const cuuint64_t strides[2] = {(cuuint64_t)kHeadDim * 2, 128};
    const cuuint32_t box[3] = {64, (cuuint32_t)kBlock, (cuuint32_t)box_chunks};
    const cuuint32_t estr[3] = {1, 1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(kcache), dims, strides,
              box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The same 3-D view of q ([total rows][576] bf16): box {64, box_rows, box_chunks}.
bool make_q_map(CUtensorMap* map, const void* q, size_t total_rows, int box_chunks,
                int box_rows = 64) {
    EncodeTiledFn fn = encode_tiled_fn();
    if (!fn) return false;
    const cuuint64_t dims[3] = {64, (cuuint64_t)total_rows, (cuuint64_t)(kHeadDim / 64)};
    const cuuint64_t strides[2] = {(cuuint64_t)kHeadDim * 2, 128};
    const cuuint32_t box[3] = {64, (cuuint32_t)box_rows, (cuuint32_t)box_chunks};
    const cuuint32_t estr[3] = {1, 1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(q), dims, strides, box,
              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

mla_status validate_decode(const uint16_t* q, const uint16_t* kcache, int num_blocks,
                           const int32_t* block_table, int max_blocks, const int32_t* seqlens,
                           int batch, int s_q, int h_q, float scale, int causal,
                           const int32_t* metadata, const int32_t* num_splits, void* workspace,
                           size_t workspace_bytes, uint16_t* out, float* lse) {
    if (!q || !kcache || !block_table || !seqlens || !metadata || !num_splits || !workspace ||
        !out || !lse)
        return MLA_ERR_INVALID_ARG;
    if (num_blocks < 1 || max_blocks < 1 || !std::isfinite(scale) || (causal != 0 && causal != 1))
        return MLA_ERR_INVALID_ARG;
    if (((uintptr_t)q | (uintptr_t)kcache | (uintptr_t)out) & 15u) return MLA_ERR_INVALID_ARG;
    if (((uintptr_t)workspace) & (kAlign - 1)) return MLA_ERR_INVALID_ARG;
    if (((uintptr_t)lse | (uintptr_t)seqlens | (uintptr_t)block_table) & 3u)
        return MLA_ERR_INVALID_ARG;
    if (!shape_ok(batch, h_q, s_q)) return MLA_ERR_UNSUPPORTED;
    if ((size_t)num_blocks * kBlock * kHeadDim * 2 >= ((size_t)1 << 47)) return MLA_ERR_UNSUPPORTED;
    if (workspace_bytes < mla_workspace_bytes(batch, h_q, s_q, 1))
        return MLA_ERR_WORKSPACE_TOO_SMALL;
    return MLA_OK;
}

DecodeParams make_params(const uint16_t* q, const uint16_t* kcache, int num_blocks,
                         const int32_t* block_table, int max_blocks, const int32_t* seqlens,
                         int batch, int s_q, int h_q, float scale, int causal,
                         const int32_t* metadata, const int32_t* num_splits, void* workspace,
                         size_t workspace_bytes, uint16_t* out, float* lse) {
    DecodeParams p;
    p.q = reinterpret_cast<const __nv_bfloat16*>(q);
    p.kcache = reinterpret_cast<const __nv_bfloat16*>(kcache);
    p.block_table = block_table;
    p.seqlens = seqlens;
    p.metadata = metadata;
    p.num_splits = num_splits;
    const size_t cap = ws_capacity(workspace_bytes);
    p.ws_lse = reinterpret_cast<float*>(static_cast<char*>(workspace) + kWsHeader);
    p.ws_o = reinterpret_cast<float*>(static_cast<char*>(workspace) + ws_o_offset(cap));
    p.max_chunks = (int)(cap > 0x7fffffff ? 0x7fffffff : cap);
    p.out = reinterpret_cast<__nv_bfloat16*>(out);
    p.lse = lse;
    p.out_f32 = nullptr;
    p.num_blocks = num_blocks;
    p.max_blocks = max_blocks;
    p.batch = batch;
    p.s_q = s_q;
    p.h_q = h_q;
    p.rows = s_q * h_q;
    p.tiles = num_tiles(h_q, s_q);
    p.scale_log2 = scale * kLog2e;
    p.causal = causal;
    return p;
}

// Device address of g_noalloc_scratch on `dev`, which must be the current device. Looked
// up on the first call for each device and cached; nullptr if the lookup fails.
void* noalloc_scratch(int dev) {
    static std::mutex mu;
    static std::vector<void*> addr;
    std::lock_guard<std::mutex> lock(mu);
    if ((int)addr.size() <= dev) addr.resize(dev + 1, nullptr);
    if (!addr[dev]) {
        void* ptr = nullptr;
        if (cudaGetSymbolAddress((void**)&ptr, g_noalloc_scratch) != cudaSuccess) {
            cudaGetLastError();
            return nullptr;
        }
        addr[dev] = ptr;
    }
    return addr[dev];
}

// Launches `kernel` with programmatic stream serialization: it may be scheduled before
// the previous kernel in the stream ends (once that kernel's blocks have all signalled
// launch_dependents) and waits for it in grid_dependency_wait().
template <class... KArgs, class... Args>
cudaError_t launch_programmatic(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                                cudaStream_t s, Args&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, args...);
}

mla_status launch_combine(const DecodeParams& p, cudaStream_t s) {
    // one warp per row of a tile; a tile of a sequence with fewer rows needs fewer CTAs
    const int tile_rows = p.rows < kTileRows ? p.rows : kTileRows;
    // slice CTAs for rows of many chunks only where the grid is small: a big grid's
    // extra CTAs, which exit at once when no row needs them, cost more than they save
    const int groups = (tile_rows + kCombineRowsPerCta - 1) / kCombineRowsPerCta;
    const size_t cells = (size_t)p.batch * p.tiles * groups;
    dim3 grid(p.batch * p.tiles, groups, cells <= (size_t)kSliceGridMax ? kCombineSlices : 1);
    combine_kernel<<<grid, kCombineThreads, 0, s>>>(p);
    return cudaGetLastError() == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

template <int kN>
mla_status launch_solo(const DecodeParams& p, const void* q, const void* kcache, int num_blocks,
                       int ctas, int dev, cudaStream_t s) {
    using C = solo::Cfg<kN>;
    if (!prepare_solo_kernel<C>(dev)) return MLA_ERR_CUDA;
    CUtensorMap tm_page, tm_q;
    if (!make_page_map(&tm_page, kcache, num_blocks, 9) ||
        !make_q_map(&tm_q, q, (size_t)p.batch * p.rows, 9, kN))
        return MLA_ERR_CUDA;
    return launch_programmatic(solo::decode_kernel<C>, dim3(ctas), dim3(C::kBlockThreads),
                               C::kSmemAlloc, s, p, tm_page, tm_page, tm_page, tm_q) == cudaSuccess
               ? MLA_OK : MLA_ERR_CUDA;
}

// FP8 cache ([num_blocks][64][656] bytes, rows of MLA_FP8_ROW_BYTES), three views a page
// lands through: the codes as a 3-D byte view {64 bytes, rows, 8 chunks} with strides {656,
// 64} and box {64, 64, 8}, so a page's 512 codes per row arrive chunk by chunk (64 rows x 64
// bytes per chunk); the scales as a 2-D byte view {16, rows} starting 512 bytes into the
// pool, box {16, 64}; the rope dims as a 2-D bf16 view {64, rows} starting 528 bytes in,
// box {64, 64}, 128-byte swizzle (one swizzled tile, as the bf16 pool's rope chunk lands).
bool make_f8_maps(CUtensorMap* codes, CUtensorMap* scales, CUtensorMap* rope, const void* kc8,
                  int num_blocks) {
    EncodeTiledFn fn = encode_tiled_fn();
    if (!fn) return false;
    const cuuint64_t rows = (cuuint64_t)num_blocks * kBlock;
    char* pool = const_cast<char*>(static_cast<const char*>(kc8));
    {
        const cuuint64_t dims[3] = {64, rows, 8};
        const cuuint64_t strides[2] = {MLA_FP8_ROW_BYTES, 64};
        const cuuint32_t box[3] = {64, (cuuint32_t)kBlock, 8};
        const cuuint32_t estr[3] = {1, 1, 1};
        if (fn(codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, pool, dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return false;
    }
    {
        const cuuint64_t dims[2] = {16, rows};
        const cuuint64_t strides[1] = {MLA_FP8_ROW_BYTES};
        const cuuint32_t box[2] = {16, (cuuint32_t)kBlock};
        const cuuint32_t estr[2] = {1, 1};
        if (fn(scales, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, pool + 512, dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return false;
    }
    {
        const cuuint64_t dims[2] = {64, rows};
        const cuuint64_t strides[1] = {MLA_FP8_ROW_BYTES};
        const cuuint32_t box[2] = {64, (cuuint32_t)kBlock};
        const cuuint32_t estr[2] = {1, 1};
        if (fn(rope, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, pool + 528, dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return false;
    }
    return true;
}

template <int kN>
mla_status launch_solo_f8(const DecodeParams& p, const void* q, const void* kc8, int num_blocks,
                          int ctas, int dev, cudaStream_t s) {
    using C = solo::Cfg<kN, true>;
    if (!prepare_solo_kernel<C>(dev)) return MLA_ERR_CUDA;
    CUtensorMap tm_codes, tm_scales, tm_rope, tm_q;
    if (!make_f8_maps(&tm_codes, &tm_scales, &tm_rope, kc8, num_blocks) ||
        !make_q_map(&tm_q, q, (size_t)p.batch * p.rows, 9, kN))
        return MLA_ERR_CUDA;
    return launch_programmatic(solo::decode_kernel<C>, dim3(ctas), dim3(C::kBlockThreads),
                               C::kSmemAlloc, s, p, tm_codes, tm_scales, tm_rope, tm_q) == cudaSuccess
               ? MLA_OK : MLA_ERR_CUDA;
}

// The split kernel for these shapes (1-CTA up to 64 rows per sequence, else 2-CTA
// pairs), then the combine. `p` is complete; q and kcache are its tensors.
mla_status launch_decode(const DecodeParams& p, const void* q, const void* kcache,
                         int num_blocks, cudaStream_t s) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return MLA_ERR_CUDA;
    mla_status st = MLA_OK;
    if (p.rows <= kSoloMaxRows) {
        const int ctas = device_solo_ctas(dev);
        if (ctas < 1) return MLA_ERR_CUDA;
        st = p.rows <= 16 ? launch_solo<16>(p, q, kcache, num_blocks, ctas, dev, s)
           : p.rows <= 32 ? launch_solo<32>(p, q, kcache, num_blocks, ctas, dev, s)
                          : launch_solo<64>(p, q, kcache, num_blocks, ctas, dev, s);
    } else {
        const int pairs = device_pairs(dev);
        if (pairs < 1 || !prepare_split_kernel(dev)) return MLA_ERR_CUDA;
        CUtensorMap tm_page, tm_pair, tm_q4, tm_q5;
        const size_t q_rows = (size_t)p.batch * p.rows;
        if (!make_page_map(&tm_page, kcache, num_blocks, 9) ||
            !make_page_map(&tm_pair, kcache, num_blocks, 2) ||
            !make_q_map(&tm_q4, q, q_rows, 4) || !make_q_map(&tm_q5, q, q_rows, 5))
            return MLA_ERR_CUDA;
        st = launch_programmatic(pair::decode_kernel, dim3(2 * pairs), dim3(pair::kThreads),
                                 pair::kSmemAlloc, s, p, tm_page, tm_pair, tm_q4, tm_q5) == cudaSuccess
                 ? MLA_OK : MLA_ERR_CUDA;
    }
    if (st != MLA_OK) return st;
    return launch_combine(p, s);
}

// mla_decode_fwd and mla_decode_fwd_partial: bf16 `out` or fp32 `out_f32` (one is null).
mla_status decode_tc(const uint16_t* q, const uint16_t* kcache, int num_blocks,
                     const int32_t* block_table, int max_blocks, const int32_t* seqlens,
                     int batch, int s_q, int h_q, float scale, int causal,
                     const int32_t* metadata, const int32_t* num_splits, void* workspace,
                     size_t workspace_bytes, uint16_t* out, float* out_f32, float* lse,
                     void* stream) {
    uint16_t* out_any = out ? out : reinterpret_cast<uint16_t*>(out_f32);
    mla_status st = validate_decode(q, kcache, num_blocks, block_table, max_blocks, seqlens,
                                    batch, s_q, h_q, scale, causal, metadata, num_splits,
                                    workspace, workspace_bytes, out_any, lse);
    if (st != MLA_OK) return st;
    DecodeParams p = make_params(q, kcache, num_blocks, block_table, max_blocks, seqlens,
                                 batch, s_q, h_q, scale, causal, metadata, num_splits,
                                 workspace, workspace_bytes, out, lse);
    p.out_f32 = out_f32;
    return launch_decode(p, q, kcache, num_blocks, (cudaStream_t)stream);
}

}  // namespace

extern "C" {

const char* mla_status_string(mla_status status) {
    switch (status) {
        case MLA_OK: return "MLA_OK";
        case MLA_ERR_INVALID_ARG: return "MLA_ERR_INVALID_ARG";
        case MLA_ERR_UNSUPPORTED: return "MLA_ERR_UNSUPPORTED";
        case MLA_ERR_CUDA: return "MLA_ERR_CUDA";
        case MLA_ERR_WORKSPACE_TOO_SMALL: return "MLA_ERR_WORKSPACE_TOO_SMALL";
        case MLA_ERR_DEVICE_TIMEOUT: return "MLA_ERR_DEVICE_TIMEOUT";
        case MLA_ERR_DEVICE_BAD_INPUT: return "MLA_ERR_DEVICE_BAD_INPUT";
        default: return "MLA_ERR_UNKNOWN";
    }
}

size_t mla_metadata_ints(int num_sms) {
    return num_sms < 1 ? 0 : (size_t)kMetaInts * ((size_t)num_sms + 1);
}

size_t mla_num_splits_len(int batch, int h_q, int s_q) {
    if (!shape_ok(batch, h_q, s_q)) return 0;
    return (size_t)batch * num_tiles(h_q, s_q) + 1;
}

size_t mla_workspace_bytes(int batch, int h_q, int s_q, int num_sms) {
    if (!shape_ok(batch, h_q, s_q) || num_sms < 1) return 0;
    return workspace_bytes_for(max_chunks_for(batch, h_q, s_q, num_sms));
}

int mla_num_work_units(int num_sms, int h_q, int s_q) {
    if (num_sms < 1) return MLA_ERR_INVALID_ARG;
    if (h_q < 1 || s_q < 1 || h_q > MLA_MAX_H_Q || s_q > MLA_MAX_S_Q || h_q * s_q > MLA_MAX_ROWS)
        return MLA_ERR_UNSUPPORTED;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return MLA_ERR_CUDA;
    const int cap = device_units(dev, h_q, s_q);
    if (cap < 1) return MLA_ERR_CUDA;
    const int u = units_bound(num_sms, h_q, s_q);
    return u > cap ? cap : u;
}

mla_status mla_test_set_stall(int stall, unsigned long long wait_limit_ns) {
    if (stall != 0 && stall != 1) return MLA_ERR_INVALID_ARG;
    const unsigned long long limit = wait_limit_ns == 0 ? 2000000000ull : wait_limit_ns;
    if (cudaMemcpyToSymbol(g_mla_debug_stall, &stall, sizeof(stall)) != cudaSuccess ||
        cudaMemcpyToSymbol(g_mla_wait_limit_ns, &limit, sizeof(limit)) != cudaSuccess)
        return MLA_ERR_CUDA;
    return MLA_OK;
}

mla_status mla_get_metadata(const int32_t* seqlens, int batch, int h_q, int s_q, int num_sms,
                            int32_t* metadata, int32_t* num_splits, void* stream) {
    if (!seqlens || !metadata || !num_splits || num_sms < 1) return MLA_ERR_INVALID_ARG;
    if (!shape_ok(batch, h_q, s_q)) return MLA_ERR_UNSUPPORTED;
    const int units = mla_num_work_units(num_sms, h_q, s_q);
    if (units < 0) return units;
    const int tiles = num_tiles(h_q, s_q);
    const size_t table = ((size_t)batch * tiles + 1 + (size_t)batch) * sizeof(int32_t);
    const bool in_smem = table <= kMetaSmemMax && prepare_metadata_kernel();
    // a small schedule is latency-bound: fewer threads mean cheaper block-wide scans
    const int threads = (size_t)batch * tiles <= 8192 ? 256 : kMetaThreads;
    metadata_kernel<<<1, threads, in_smem ? table : 0, (cudaStream_t)stream>>>(
        seqlens, batch, h_q, s_q, tiles, units, in_smem ? 1 : 0, metadata, num_splits);
    return cudaGetLastError() == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

mla_status mla_decode_fwd_simt(const uint16_t* q, const uint16_t* kcache, int num_blocks,
                               const int32_t* block_table, int max_blocks,
                               const int32_t* seqlens, int batch, int s_q, int h_q,
                               float scale, int causal, const int32_t* metadata,
                               const int32_t* num_splits, void* workspace,
                               size_t workspace_bytes, uint16_t* out, float* lse,
                               void* stream) {
    mla_status st = validate_decode(q, kcache, num_blocks, block_table, max_blocks, seqlens,
                                    batch, s_q, h_q, scale, causal, metadata, num_splits,
                                    workspace, workspace_bytes, out, lse);
    if (st != MLA_OK) return st;
    DecodeParams p = make_params(q, kcache, num_blocks, block_table, max_blocks, seqlens,
                                 batch, s_q, h_q, scale, causal, metadata, num_splits,
                                 workspace, workspace_bytes, out, lse);
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return MLA_ERR_CUDA;
    const int units = device_units(dev, h_q, s_q);
    if (units < 1) return MLA_ERR_CUDA;
    cudaStream_t s = (cudaStream_t)stream;
    decode_simt_kernel<<<units, kSimtThreads, 0, s>>>(p);
    if (cudaGetLastError() != cudaSuccess) return MLA_ERR_CUDA;
    return launch_combine(p, s);
}

mla_status mla_decode_fwd(const uint16_t* q, const uint16_t* kcache, int num_blocks,
                          const int32_t* block_table, int max_blocks, const int32_t* seqlens,
                          int batch, int s_q, int h_q, float scale, int causal,
                          const int32_t* metadata, const int32_t* num_splits, void* workspace,
                          size_t workspace_bytes, uint16_t* out, float* lse, void* stream) {
    return decode_tc(q, kcache, num_blocks, block_table, max_blocks, seqlens, batch, s_q, h_q,
                     scale, causal, metadata, num_splits, workspace, workspace_bytes, out,
                     nullptr, lse, stream);
}

mla_status mla_decode_fwd_partial(const uint16_t* q, const uint16_t* kcache, int num_blocks,
                                  const int32_t* block_table, int max_blocks,
                                  const int32_t* seqlens, int batch, int s_q, int h_q,
                                  float scale, int causal, const int32_t* metadata,
                                  const int32_t* num_splits, void* workspace,
                                  size_t workspace_bytes, float* out_f32, float* lse,
                                  void* stream) {
    return decode_tc(q, kcache, num_blocks, block_table, max_blocks, seqlens, batch, s_q, h_q,
                     scale, causal, metadata, num_splits, workspace, workspace_bytes, nullptr,
                     out_f32, lse, stream);
}

mla_status mla_combine_partials(const float* o_parts, const float* lse_parts, int parts,
                                int batch, int s_q, int h_q, uint16_t* out, float* lse,
                                void* stream) {
    if (!o_parts || !lse_parts || !out || !lse || parts < 1 || parts > MLA_MAX_PARTS)
        return MLA_ERR_INVALID_ARG;
    if (((uintptr_t)o_parts | (uintptr_t)out) & 15u) return MLA_ERR_INVALID_ARG;
    if (((uintptr_t)lse_parts | (uintptr_t)lse) & 3u) return MLA_ERR_INVALID_ARG;
    if (!shape_ok(batch, h_q, s_q)) return MLA_ERR_UNSUPPORTED;
    RankCombineParams p;
    p.o_parts = o_parts;
    p.lse_parts = lse_parts;
    p.out = reinterpret_cast<__nv_bfloat16*>(out);
    p.lse = lse;
    p.parts = parts;
    p.batch = batch;
    p.s_q = s_q;
    p.h_q = h_q;
    const long long rows = (long long)batch * s_q * h_q;
    const unsigned grid = (unsigned)((rows + kRankCombineRowsPerCta - 1) / kRankCombineRowsPerCta);
    rank_combine_kernel<<<grid, kRankCombineThreads, 0, (cudaStream_t)stream>>>(p);
    return cudaGetLastError() == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

mla_status mla_decode_fwd_noalloc(const uint16_t* q, const uint16_t* kcache, int num_blocks,
                                  const int32_t* block_table, int max_blocks,
                                  const int32_t* seqlens, int batch, int s_q, int h_q,
                                  float scale, int causal, const int32_t* metadata,
                                  const int32_t* num_splits, uint16_t* out, float* lse,
                                  void* stream) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return MLA_ERR_CUDA;
    void* scratch = noalloc_scratch(dev);
    if (!scratch) return MLA_ERR_CUDA;
    const size_t scratch_bytes = MLA_NOALLOC_SCRATCH_BYTES;
    mla_status st = validate_decode(q, kcache, num_blocks, block_table, max_blocks, seqlens,
                                    batch, s_q, h_q, scale, causal, metadata, num_splits,
                                    scratch, scratch_bytes, out, lse);
    if (st != MLA_OK) return st;
    const int units = device_units(dev, h_q, s_q);
    if (units < 1) return MLA_ERR_CUDA;
    // worst case over every schedule this device can run: one chunk per work sequence
    // plus one per unit
    if (workspace_bytes_for((size_t)batch * num_tiles(h_q, s_q) + (size_t)units) > scratch_bytes)
        return MLA_ERR_WORKSPACE_TOO_SMALL;
    DecodeParams p = make_params(q, kcache, num_blocks, block_table, max_blocks, seqlens,
                                 batch, s_q, h_q, scale, causal, metadata, num_splits,
                                 scratch, scratch_bytes, out, lse);
    return launch_decode(p, q, kcache, num_blocks, (cudaStream_t)stream);
}

mla_status mla_decode_fwd_fp8(const uint16_t* q, const uint8_t* kcache_fp8, int num_blocks,
                              const int32_t* block_table, int max_blocks, const int32_t* seqlens,
                              int batch, int s_q, int h_q, float scale, int causal,
                              const int32_t* metadata, const int32_t* num_splits,
                              void* workspace, size_t workspace_bytes, uint16_t* out, float* lse,
                              void* stream) {
    // the validation of mla_decode_fwd (the cache pointer takes the bf16 pool's checks)
    mla_status st = validate_decode(q, reinterpret_cast<const uint16_t*>(kcache_fp8), num_blocks,
                                    block_table, max_blocks, seqlens, batch, s_q, h_q, scale,
                                    causal, metadata, num_splits, workspace, workspace_bytes, out,
                                    lse);
    if (st != MLA_OK) return st;
    if (h_q * s_q > kFp8MaxRows) return MLA_ERR_UNSUPPORTED;
    DecodeParams p = make_params(q, reinterpret_cast<const uint16_t*>(kcache_fp8), num_blocks,
                                 block_table, max_blocks, seqlens, batch, s_q, h_q, scale, causal,
                                 metadata, num_splits, workspace, workspace_bytes, out, lse);
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return MLA_ERR_CUDA;
    const int ctas = device_solo_ctas(dev);
    if (ctas < 1) return MLA_ERR_CUDA;
    cudaStream_t s = (cudaStream_t)stream;
    st = p.rows <= 16 ? launch_solo_f8<16>(p, q, kcache_fp8, num_blocks, ctas, dev, s)
       : p.rows <= 32 ? launch_solo_f8<32>(p, q, kcache_fp8, num_blocks, ctas, dev, s)
                      : launch_solo_f8<64>(p, q, kcache_fp8, num_blocks, ctas, dev, s);
    if (st != MLA_OK) return st;
    return launch_combine(p, s);
}

mla_status mla_kv_append(const uint16_t* kv_new, int s_new, const int32_t* block_table,
                         int max_blocks, const int32_t* seqlens, int batch, uint16_t* kcache,
                         int num_blocks, void* stream) {
    if (!kv_new || !block_table || !seqlens || !kcache) return MLA_ERR_INVALID_ARG;
    if (num_blocks < 1 || max_blocks < 1 || s_new < 1) return MLA_ERR_INVALID_ARG;
    if (((uintptr_t)kv_new | (uintptr_t)kcache) & 15u) return MLA_ERR_INVALID_ARG;
    if (((uintptr_t)block_table | (uintptr_t)seqlens) & 3u) return MLA_ERR_INVALID_ARG;
    if (batch < 1 || batch > MLA_MAX_BATCH || s_new > MLA_MAX_S_Q) return MLA_ERR_UNSUPPORTED;
    const long long rows = (long long)batch * s_new;
    const int per_cta = kAppendThreads / 32;
    const unsigned grid = (unsigned)((rows + per_cta - 1) / per_cta);
    kv_append_kernel<<<grid, kAppendThreads, 0, (cudaStream_t)stream>>>(
        reinterpret_cast<const uint4*>(kv_new), s_new, block_table, max_blocks, seqlens, batch,
        reinterpret_cast<uint4*>(kcache), num_blocks);
    return cudaGetLastError() == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

mla_status mla_kv_append_fp8(const uint16_t* kv_new, int s_new, const int32_t* block_table,
                             int max_blocks, const int32_t* seqlens, int batch,
                             uint8_t* kcache_fp8, int num_blocks, void* stream) {
    if (!kv_new || !block_table || !seqlens || !kcache_fp8) return MLA_ERR_INVALID_ARG;
    if (num_blocks < 1 || max_blocks < 1 || s_new < 1) return MLA_ERR_INVALID_ARG;
    if (((uintptr_t)kv_new | (uintptr_t)kcache_fp8) & 15u) return MLA_ERR_INVALID_ARG;
    if (((uintptr_t)block_table | (uintptr_t)seqlens) & 3u) return MLA_ERR_INVALID_ARG;
    if (batch < 1 || batch > MLA_MAX_BATCH || s_new > MLA_MAX_S_Q) return MLA_ERR_UNSUPPORTED;
    const long long rows = (long long)batch * s_new;
    const int per_cta = kAppendThreads / 32;
    const unsigned grid = (unsigned)((rows + per_cta - 1) / per_cta);
    kv_append_fp8_kernel<<<grid, kAppendThreads, 0, (cudaStream_t)stream>>>(
        reinterpret_cast<const __nv_bfloat16*>(kv_new), s_new, block_table, max_blocks, seqlens,
        batch, kcache_fp8, num_blocks);
    return cudaGetLastError() == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

mla_status mla_get_last_device_error(void* stream, uint32_t* detail) {
    if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return MLA_ERR_CUDA;
    uint32_t w = 0;
    if (cudaMemcpyFromSymbol(&w, g_mla_error, sizeof(w)) != cudaSuccess) return MLA_ERR_CUDA;
    if (detail) *detail = w;
    if (w == 0) return MLA_OK;
    const uint32_t zero = 0;
    if (cudaMemcpyToSymbol(g_mla_error, &zero, sizeof(zero)) != cudaSuccess) return MLA_ERR_CUDA;
    return (w & 0xffu) == kErrTimeout ? MLA_ERR_DEVICE_TIMEOUT : MLA_ERR_DEVICE_BAD_INPUT;
}

mla_status mla_plan_host(const int32_t* seqlens_host, int batch, int h_q, int s_q,
                         int num_units, int32_t* metadata_host, int32_t* num_splits_host) {
    if (!seqlens_host || !metadata_host || !num_splits_host || num_units < 1)
        return MLA_ERR_INVALID_ARG;
    if (!shape_ok(batch, h_q, s_q)) return MLA_ERR_UNSUPPORTED;
    const int tiles = num_tiles(h_q, s_q);
    const int V = batch * tiles;
    const int overhead = overhead_pages(h_q, s_q);
    std::vector<int> nblk(V);
    std::vector<int64_t> C(V + 1, 0);
    for (int v = 0; v < V; ++v) {
        const int L = seqlens_host[v % batch];
        nblk[v] = pages_of(L < 0 ? 0 : L);
        C[v + 1] = C[v] + overhead + nblk[v];
    }
    if (C[V] > 0x7fffffffLL) return MLA_ERR_UNSUPPORTED;
    auto cost = [&](int v) { return C[v]; };
    auto pages = [&](int v) { return nblk[v]; };
    const int64_t W = header_unit_cost(num_units, tiles, batch, V, cost);
    for (int u = 0; u < num_units; ++u) {
        int vb, kb, ve, ke, chunk;
        unit_range(u, num_units, tiles, batch, V, overhead, cost, pages, &vb, &kb, &ve, &ke, &chunk);
        int32_t* m = metadata_host + kMetaInts * (u + 1);
        m[0] = vb; m[1] = kb; m[2] = ve; m[3] = ke; m[4] = chunk;
        m[5] = 0; m[6] = 0; m[7] = 0;
    }
    metadata_host[0] = num_units; metadata_host[1] = tiles; metadata_host[2] = batch;
    metadata_host[3] = h_q; metadata_host[4] = s_q; metadata_host[5] = (int32_t)W;
    metadata_host[6] = overhead; metadata_host[7] = tile_aligned(tiles, num_units) ? 1 : 0;
    int32_t acc = 0;
    for (int v = 0; v < V; ++v) {
        num_splits_host[v] = acc;
        acc += chunks_of_v(v, num_units, tiles, batch, V, overhead, cost, pages);
    }
    num_splits_host[V] = acc;
    return MLA_OK;
}

}  // extern "C"
