// pagedkv.cu -- host side of libpagedkv.so: argument checks, TMA tensor maps,
// kernel selection and launches behind the C ABI of include/pagedkv.h.
//
// The library is one translation unit (the kernels live in the .cuh files
// included below) so that all kernels share the device error word.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <set>
#include <vector>

#include "pagedkv.h"
#include "ptx.cuh"
#include "index_kernels.cuh"
#include "decode.cuh"
#include "decode_mma.cuh"
#include "decode_fp8.cuh"
#include "decode_multi.cuh"
#include "prefill.cuh"

namespace {

thread_local char g_last_cuda_error[256] = "";

int cuda_fail(cudaError_t e, const char* where) {
    snprintf(g_last_cuda_error, sizeof g_last_cuda_error, "%s: %s", where, cudaGetErrorString(e));
    return PKV_ECUDA;
}

#define PKV_CUDA(call)                                      \
    do {                                                    \
        cudaError_t e__ = (call);                           \
        if (e__ != cudaSuccess) return cuda_fail(e__, #call); \
    } while (0)

int elem_bytes(int dtype) {
    switch (dtype) {
        case PKV_F32: return 4;
        case PKV_F16: return 2;
        case PKV_BF16: return 2;
        case PKV_FP8_E4M3: return 1;
        default: return 0;
    }
}

// Types a query / output may have (FP8 is a pool type only).
bool query_type(int dtype) { return dtype == PKV_F32 || dtype == PKV_F16 || dtype == PKV_BF16; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

bool checked_mode() {
    static const bool on = [] {
        const char* v = getenv("PKV_CHECK");
        return v && v[0] && strcmp(v, "0") != 0;
    }();
    return on;
}

// ------------------------------------------------------------ tensor maps
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

CUtensorMapDataType cu_type(int dtype) {
    switch (dtype) {
        case PKV_F32: return CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
        case PKV_F16: return CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
        case PKV_FP8_E4M3: return CU_TENSOR_MAP_DATA_TYPE_UINT8;
        default: return CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    }
}

// Pool [num_blocks, block_size, num_kv_heads, head_dim] as a 4-D tensor
// (head_dim innermost); one box = one block x one KV head x 128 bytes of
// head_dim, 128-byte swizzled.
// box_rows: tokens per box (the whole block by default).
int make_pool_map(CUtensorMap* map, const void* pool, int dtype, int64_t num_blocks, int block_size,
                  int num_kv_heads, int head_dim, int box_rows = 0) {
    auto fn = encode_fn();
    if (!fn) {
        snprintf(g_last_cuda_error, sizeof g_last_cuda_error, "cuTensorMapEncodeTiled unavailable");
        return PKV_ECUDA;
    }
    const int eb = elem_bytes(dtype);
    cuuint64_t dims[4] = {(cuuint64_t)head_dim, (cuuint64_t)num_kv_heads, (cuuint64_t)block_size,
                          (cuuint64_t)num_blocks};
    cuuint64_t strides[3] = {(cuuint64_t)head_dim * eb, (cuuint64_t)num_kv_heads * head_dim * eb,
                             (cuuint64_t)block_size * num_kv_heads * head_dim * eb};
    cuuint32_t box[4] = {(cuuint32_t)(128 / eb), 1, (cuuint32_t)(box_rows > 0 ? box_rows : block_size), 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = fn(map, cu_type(dtype), 4, const_cast<void*>(pool), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        snprintf(g_last_cuda_error, sizeof g_last_cuda_error, "cuTensorMapEncodeTiled(pool) failed: %d", (int)r);
        return PKV_ECUDA;
    }
    return PKV_OK;
}

// Packed query [tokens, num_q_heads, head_dim] as a 3-D tensor; one box =
// box_tokens (default 128 / group) tokens x group heads x 128 bytes of head_dim.
int make_query_map(CUtensorMap* map, const void* q, int dtype, int64_t tokens, int num_q_heads, int head_dim,
                   int group, int box_tokens = 0) {
    auto fn = encode_fn();
    if (!fn) {
        snprintf(g_last_cuda_error, sizeof g_last_cuda_error, "cuTensorMapEncodeTiled unavailable");
        return PKV_ECUDA;
    }
    const int eb = elem_bytes(dtype);
    cuuint64_t dims[3] = {(cuuint64_t)head_dim, (cuuint64_t)num_q_heads, (cuuint64_t)tokens};
    cuuint64_t strides[2] = {(cuuint64_t)head_dim * eb, (cuuint64_t)num_q_heads * head_dim * eb};
    cuuint32_t box[3] = {(cuuint32_t)(128 / eb), (cuuint32_t)group,
                         (cuuint32_t)(box_tokens > 0 ? box_tokens : 128 / group)};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(map, cu_type(dtype), 3, const_cast<void*>(q), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        snprintf(g_last_cuda_error, sizeof g_last_cuda_error, "cuTensorMapEncodeTiled(query) failed: %d", (int)r);
        return PKV_ECUDA;
    }
    return PKV_OK;
}

int sm_count() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
    return n;
}

// ------------------------------------------------------------ checked mode
template <typename I>
int fetch(std::vector<I>& host, const I* dev, size_t n, cudaStream_t s) {
    host.resize(n);
    if (n == 0) return PKV_OK;
    PKV_CUDA(cudaMemcpyAsync(host.data(), dev, n * sizeof(I), cudaMemcpyDeviceToHost, s));
    PKV_CUDA(cudaStreamSynchronize(s));
    return PKV_OK;
}

int check_tables(const int32_t* d_bt, const int32_t* d_lens, int num_seqs, int max_blocks, int block_size,
                 int64_t num_blocks, int64_t max_len, cudaStream_t s) {
    std::vector<int32_t> bt, lens;
    int rc = fetch(lens, d_lens, num_seqs, s);
    if (rc) return rc;
    rc = fetch(bt, d_bt, (size_t)num_seqs * max_blocks, s);
    if (rc) return rc;
    for (int i = 0; i < num_seqs; ++i) {
        const int64_t n = lens[i];
        if (n < 0 || n > max_len || n > (int64_t)max_blocks * block_size) return PKV_ERANGE;
        const int64_t nb = (n + block_size - 1) / block_size;
        for (int64_t b = 0; b < nb; ++b) {
            const int32_t id = bt[(size_t)i * max_blocks + b];
            if (id < 0 || id >= num_blocks) return PKV_ERANGE;
        }
    }
    return PKV_OK;
}

// ------------------------------------------------------------ launches
// Stream of a launch and whether the kernel may start as a programmatic
// dependent of the kernel before it in the stream (its prologue overlapping
// that kernel's tail; the kernel waits with griddepcontrol.wait before it
// touches what that kernel writes).
struct Launch {
    cudaStream_t s;
    bool pdl;
};

template <typename... KArgs, typename... Args>
int launch_kernel(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, const Launch& ln, Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = ln.s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = ln.pdl ? 1 : 0;
    PKV_CUDA(cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...));
    PKV_CUDA(cudaGetLastError());
    return PKV_OK;
}

// ------------------------------------------------------------ decode dispatch
// Launch shape of the decode kernels, from a sweep on B200 of warps per CTA x
// stages per warp at equal shared memory: 8 KB stages (block 16, 16-bit,
// head_dim 128) run best as 4 warps x 2 stages (64 KB, three CTAs per SM);
// 16 KB stages as 8 warps x 1 stage (one CTA per SM).
#ifndef PKV_DECODE_STAGE_BUDGET
#define PKV_DECODE_STAGE_BUDGET 65536  // bytes of K/V stages per 4-warp decode CTA
#endif

constexpr int pick_warps(int stage_bytes) { return (stage_bytes >= 16384 && 8 * stage_bytes <= 160 * 1024) ? 8 : 4; }

constexpr int pick_stages(int stage_bytes, int warps) {
    int n = (warps == 8 ? 2 * PKV_DECODE_STAGE_BUDGET : PKV_DECODE_STAGE_BUDGET) / (warps * stage_bytes);
    if (n < 1) n = 1;
    if (n > 4) n = 4;
    return n;
}

template <typename Kern>
int launch_decode_kernel(Kern kern, size_t smem, int threads, const pkv::DecodeParams& prm, const CUtensorMap& tk,
                         const CUtensorMap& tv, int grid, const Launch& ln, size_t* configured) {
    int dev = 0;
    PKV_CUDA(cudaGetDevice(&dev));
    size_t& have = configured[dev & 63];  // largest dynamic smem size set so far on this device
    if (smem > have) {
        PKV_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
        have = smem;
    }
    return launch_kernel(kern, dim3(grid), dim3(threads), smem, ln, prm, tk, tv);
}

template <typename T, int D, int B, int G>
int launch_decode(const pkv::DecodeParams& prm, const CUtensorMap& tk, const CUtensorMap& tv, int grid,
                  const Launch& ln) {
    constexpr int STAGE = 2 * B * D * pkv::Elem<T>::kBytes;
#ifdef PKV_DECODE_WARPS
    constexpr int NW = PKV_DECODE_WARPS;
#else
    constexpr int NW = pick_warps(STAGE);
#endif
    constexpr int NST = pick_stages(STAGE, NW);
    using C = pkv::DecodeCfg<T, D, B, G, NST, NW>;
    const size_t smem = C::smem_bytes(prm.partition_blocks);
    static size_t configured[64] = {};
    // 16-bit types run the Q.K / P.V products on warp MMAs (one head per KV
    // head included: measured 6.6 vs 6.2 TB/s on the llama7b batch); fp32
    // stays on the CUDA cores.
#ifndef PKV_DECODE_MMA_MIN_G
#define PKV_DECODE_MMA_MIN_G 1  // 16-bit types with at least this many heads per KV head use warp MMAs
#endif
    if constexpr (sizeof(T) == 2 && G >= PKV_DECODE_MMA_MIN_G)
        return launch_decode_kernel(pkv::paged_decode_mma_kernel<T, D, B, G, NST, NW>, smem, NW * 32, prm, tk, tv,
                                    grid, ln, configured);
    else
        return launch_decode_kernel(pkv::paged_decode_kernel<T, D, B, G, NST, NW>, smem, NW * 32, prm, tk, tv,
                                    grid, ln, configured);
}

template <typename T, int D, int B>
int decode_by_group(int group, const pkv::DecodeParams& prm, const CUtensorMap& tk, const CUtensorMap& tv,
                    int grid, const Launch& ln) {
    switch (group) {
        case 1: return launch_decode<T, D, B, 1>(prm, tk, tv, grid, ln);
        case 2: return launch_decode<T, D, B, 2>(prm, tk, tv, grid, ln);
        case 4: return launch_decode<T, D, B, 4>(prm, tk, tv, grid, ln);
        case 8: return launch_decode<T, D, B, 8>(prm, tk, tv, grid, ln);
        default: return PKV_EUNSUPPORTED;
    }
}

template <typename T, int D>
int decode_by_block(int block_size, int group, const pkv::DecodeParams& prm, const CUtensorMap& tk,
                    const CUtensorMap& tv, int grid, const Launch& ln) {
    switch (block_size) {
        case 8: return decode_by_group<T, D, 8>(group, prm, tk, tv, grid, ln);
        case 16: return decode_by_group<T, D, 16>(group, prm, tk, tv, grid, ln);
        case 32: return decode_by_group<T, D, 32>(group, prm, tk, tv, grid, ln);
        default: return PKV_EUNSUPPORTED;
    }
}

template <typename T>
int decode_by_dim(int head_dim, int block_size, int group, const pkv::DecodeParams& prm, const CUtensorMap& tk,
                  const CUtensorMap& tv, int grid, const Launch& ln) {
    switch (head_dim) {
        case 64: return decode_by_block<T, 64>(block_size, group, prm, tk, tv, grid, ln);
        case 128: return decode_by_block<T, 128>(block_size, group, prm, tk, tv, grid, ln);
        default: return PKV_EUNSUPPORTED;
    }
}

#ifndef PKV_FP8_WARPS
#define PKV_FP8_WARPS 4
#endif
#ifndef PKV_FP8_UNIT_TOKENS
#define PKV_FP8_UNIT_TOKENS 32  // tokens per softmax step of the E4M3 decode with grouped heads
#endif
#ifndef PKV_FP8_STAGE_BUDGET
#define PKV_FP8_STAGE_BUDGET 32768  // bytes of K/V stages per FP8 decode CTA
#endif

template <typename T, int B, int G>
int launch_decode_fp8(const pkv::DecodeParams& prm, const CUtensorMap& tk, const CUtensorMap& tv, int grid,
                      const Launch& ln) {
    // Blocks of 8 or 16 tokens are grouped into 32-token units for 4 or 8
    // heads per KV head (+3 % on the gqa70b-shaped E4M3 batch, with twice the
    // stage budget to keep two stages per warp; no gain with one head).
    constexpr int U = (G >= 4 && B < PKV_FP8_UNIT_TOKENS) ? PKV_FP8_UNIT_TOKENS / B : 1;  // blocks per unit
    constexpr int STAGE = 2 * B * U * 128;
    constexpr int NW = PKV_FP8_WARPS;
    constexpr int NST = std::max(1, std::min(8, (U > 1 ? 2 : 1) * PKV_FP8_STAGE_BUDGET / (NW * STAGE)));
    using C = pkv::DecodeFp8Cfg<B, G, NST, NW, U>;
    static size_t configured[64] = {};
    return launch_decode_kernel(pkv::paged_decode_fp8_kernel<T, B, G, NST, NW, U>, C::smem_bytes(prm.partition_blocks),
                                NW * 32, prm, tk, tv, grid, ln, configured);
}

template <typename T, int B>
int decode_fp8_by_group(int group, const pkv::DecodeParams& prm, const CUtensorMap& tk, const CUtensorMap& tv,
                        int grid, const Launch& ln) {
    switch (group) {
        case 1: return launch_decode_fp8<T, B, 1>(prm, tk, tv, grid, ln);
        case 2: return launch_decode_fp8<T, B, 2>(prm, tk, tv, grid, ln);
        case 4: return launch_decode_fp8<T, B, 4>(prm, tk, tv, grid, ln);
        case 8: return launch_decode_fp8<T, B, 8>(prm, tk, tv, grid, ln);
        default: return PKV_EUNSUPPORTED;
    }
}

template <typename T>
int decode_fp8_by_block(int block_size, int group, const pkv::DecodeParams& prm, const CUtensorMap& tk,
                        const CUtensorMap& tv, int grid, const Launch& ln) {
    switch (block_size) {
        case 8: return decode_fp8_by_group<T, 8>(group, prm, tk, tv, grid, ln);
        case 16: return decode_fp8_by_group<T, 16>(group, prm, tk, tv, grid, ln);
        case 32: return decode_fp8_by_group<T, 32>(group, prm, tk, tv, grid, ln);
        default: return PKV_EUNSUPPORTED;
    }
}

// ------------------------------------------------------------ multi-token decode dispatch
// Persistent: as many CTAs as fit on the device at once (one per SM at
// head_dim 128), at most one per item.
template <typename T, int D>
int launch_multi(const pkv::MultiParams& prm, int lpt, const CUtensorMap& tq, const CUtensorMap& tk,
                 const CUtensorMap& tv, int64_t items, const Launch& ln) {
    using C = pkv::MultiCfg<D>;
    auto kern = pkv::paged_decode_multi_kernel<T, D>;
    int dev = 0;
    PKV_CUDA(cudaGetDevice(&dev));
    static int resident[64] = {};  // CTAs per SM, per device (0: not configured yet)
    int& per_sm = resident[dev & 63];
    if (per_sm == 0) {
        PKV_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM));
        int n = 0;
        PKV_CUDA(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, pkv::kMultiThreads, C::SMEM));
        if (n <= 0) return PKV_EUNSUPPORTED;
        per_sm = n;
    }
    const int grid = (int)std::min<int64_t>(items, (int64_t)sm_count() * per_sm);
    return launch_kernel(kern, dim3(grid), dim3(pkv::kMultiThreads), C::SMEM, ln, prm, lpt, tq, tk, tv);
}

// The merge always follows this library's own decode kernel in the stream,
// so it is launched as that kernel's programmatic dependent (it waits for the
// partials before it reads them).
template <typename T>
int launch_merge(int head_dim, const pkv::MergeParams& mp, cudaStream_t s) {
    const int warps = mp.num_seqs * mp.num_q_heads;
    const int grid = (warps + 3) / 4;
    const Launch ln{s, true};
    if (head_dim == 64) return launch_kernel(pkv::paged_decode_merge_kernel<T, 64>, dim3(grid), dim3(128), 0, ln, mp);
    return launch_kernel(pkv::paged_decode_merge_kernel<T, 128>, dim3(grid), dim3(128), 0, ln, mp);
}

bool supported_group(int g) { return g == 1 || g == 2 || g == 4 || g == 8; }

// A decode CTA keeps its partition's block ids in shared memory: at most this
// many blocks per partition.
constexpr int64_t kMaxPartitionBlocks = 4096;

int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

// ------------------------------------------------------------ prefill dispatch
template <typename T, int D, int G, typename TO = T>
int launch_prefill(const pkv::PrefillParams& prm, const CUtensorMap& tq, const CUtensorMap& tk,
                   const CUtensorMap& tv, int grid, cudaStream_t s) {
    using C = pkv::PrefillCfg<T, D, G>;
    auto kern = pkv::paged_prefill_kernel<T, D, G, TO>;
    int dev = 0;
    PKV_CUDA(cudaGetDevice(&dev));
    static bool configured[64] = {};
    if (!configured[dev & 63]) {
        PKV_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM));
        configured[dev & 63] = true;
    }
    kern<<<grid, pkv::kPrefillThreads, C::SMEM, s>>>(prm, tq, tk, tv);
    PKV_CUDA(cudaGetLastError());
    return PKV_OK;
}

template <typename T, int D, typename TO = T>
int prefill_by_group(int group, const pkv::PrefillParams& prm, const CUtensorMap& tq, const CUtensorMap& tk,
                     const CUtensorMap& tv, int grid, cudaStream_t s) {
    switch (group) {
        case 1: return launch_prefill<T, D, 1, TO>(prm, tq, tk, tv, grid, s);
        case 2: return launch_prefill<T, D, 2, TO>(prm, tq, tk, tv, grid, s);
        case 4: return launch_prefill<T, D, 4, TO>(prm, tq, tk, tv, grid, s);
        case 8: return launch_prefill<T, D, 8, TO>(prm, tq, tk, tv, grid, s);
        default: return PKV_EUNSUPPORTED;
    }
}

// Argument checks of the decode entry points that need no workspace: the
// status the decode returns for these arguments, or PKV_OK (num_seqs == 0
// passes: it launches nothing).
int decode_check(const void* out, const void* query, const void* key_cache, const void* value_cache,
                 const int32_t* block_tables, const int32_t* context_lens, float scale, int num_seqs,
                 int num_q_heads, int num_kv_heads, int head_dim, int block_size, int max_blocks_per_seq,
                 int64_t num_blocks, int max_context_len, int partition_size, int dtype, int kv_dtype) {
    const bool fp8 = kv_dtype == PKV_FP8_E4M3;
    if (!query_type(dtype) || (kv_dtype != dtype && !fp8)) return PKV_EUNSUPPORTED;
    if (fp8 && (dtype == PKV_F32 || head_dim != 128)) return PKV_EUNSUPPORTED;
    if (num_seqs < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || max_blocks_per_seq <= 0 || num_blocks <= 0 ||
        max_context_len < 0 || partition_size < 0 || !std::isfinite(scale))
        return PKV_EINVAL;
    if (num_q_heads % num_kv_heads) return PKV_EINVAL;
    const int group = num_q_heads / num_kv_heads;
    if (!supported_group(group) || (head_dim != 64 && head_dim != 128) ||
        (block_size != 8 && block_size != 16 && block_size != 32))
        return PKV_EUNSUPPORTED;
    if (partition_size % block_size) return PKV_EINVAL;
    if (num_blocks >= (int64_t)INT32_MAX || (int64_t)max_blocks_per_seq * block_size > INT32_MAX) return PKV_EINVAL;
    if (num_seqs == 0) return PKV_OK;
    if (!out || !query || !key_cache || !value_cache || !block_tables || !context_lens) return PKV_EINVAL;
    if (!aligned16(out) || !aligned16(query) || !aligned16(key_cache) || !aligned16(value_cache) ||
        (reinterpret_cast<uintptr_t>(block_tables) & 3) || (reinterpret_cast<uintptr_t>(context_lens) & 3))
        return PKV_EINVAL;
    const int64_t max_blocks_needed = std::max<int64_t>(1, ceil_div(std::max(max_context_len, 1), block_size));
    const int64_t pb = std::min<int64_t>(partition_size > 0 ? partition_size / block_size : max_blocks_needed,
                                         max_blocks_needed);
    if (pb > kMaxPartitionBlocks) return PKV_EUNSUPPORTED;
    return PKV_OK;
}

// The workspace and grid checks of the decode (arguments already passed
// decode_check): PKV_EWORKSPACE when the split-K partials do not fit.
int decode_workspace_check(int num_seqs, int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                           int max_context_len, int partition_size, const void* workspace, size_t workspace_bytes) {
    if (num_seqs == 0) return PKV_OK;
    const int64_t max_blocks_needed = std::max<int64_t>(1, ceil_div(std::max(max_context_len, 1), block_size));
    const int64_t pb = std::min<int64_t>(partition_size > 0 ? partition_size / block_size : max_blocks_needed,
                                         max_blocks_needed);
    const int64_t parts = ceil_div(max_blocks_needed, pb);
    const size_t need = parts > 1 ? pkv_decode_workspace_size(num_seqs, num_q_heads, head_dim, max_context_len,
                                                              (int)(pb * block_size))
                                  : 0;
    if (need > 0 && (!workspace || workspace_bytes < need || !aligned16(workspace))) return PKV_EWORKSPACE;
    if ((int64_t)num_seqs * parts * num_kv_heads > INT32_MAX) return PKV_EUNSUPPORTED;
    return PKV_OK;
}

// Argument checks of the appends (16/32-bit pools, and E4M3 pools written
// from `dtype`): the status the append returns, or PKV_OK (also for
// num_tokens == 0, which launches nothing).
int reshape_check(const void* key, const void* value, const void* key_cache, const void* value_cache,
                  const int64_t* slot_mapping, int64_t num_tokens, int num_kv_heads, int head_dim, int block_size,
                  int64_t num_blocks, int dtype, bool fp8) {
    if (fp8 ? !query_type(dtype) : !elem_bytes(dtype)) return PKV_EUNSUPPORTED;
    if (num_tokens < 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 || num_blocks <= 0)
        return PKV_EINVAL;
    const int64_t row_elems = (int64_t)num_kv_heads * head_dim;
    if (fp8) {
        if (row_elems % 16 != 0 || row_elems > INT32_MAX) return PKV_EUNSUPPORTED;
    } else {
        const int64_t row_bytes = row_elems * elem_bytes(dtype);
        if (row_bytes % 16 != 0 || row_bytes / 16 > INT32_MAX) return PKV_EUNSUPPORTED;
    }
    if (num_tokens == 0) return PKV_OK;
    if (!key || !value || !key_cache || !value_cache || !slot_mapping) return PKV_EINVAL;
    if (!aligned16(key) || !aligned16(value) || !aligned16(key_cache) || !aligned16(value_cache) ||
        (reinterpret_cast<uintptr_t>(slot_mapping) & 7))
        return PKV_EINVAL;
    return PKV_OK;
}

int reshape_fp8_check(const void* key, const void* value, const void* key_cache, const void* value_cache,
                      const int64_t* slot_mapping, int64_t num_tokens, int num_kv_heads, int head_dim, int block_size,
                      int64_t num_blocks, int src_dtype) {
    return reshape_check(key, value, key_cache, value_cache, slot_mapping, num_tokens, num_kv_heads, head_dim,
                         block_size, num_blocks, src_dtype, true);
}

// Decode with the query / output in `dtype` and the pools in `kv_dtype`
// (the same 16/32-bit type, or FP8 E4M3 with its two scales).
int decode_impl(void* out, const void* query, const void* key_cache, const void* value_cache,
                const int32_t* block_tables, const int32_t* context_lens, float scale, int num_seqs, int num_q_heads,
                int num_kv_heads, int head_dim, int block_size, int max_blocks_per_seq, int64_t num_blocks,
                int max_context_len, int partition_size, int dtype, int kv_dtype, float k_scale, float v_scale,
                void* workspace, size_t workspace_bytes, pkv_stream_t stream, bool pdl = false) {
    const int check = decode_check(out, query, key_cache, value_cache, block_tables, context_lens, scale, num_seqs,
                                   num_q_heads, num_kv_heads, head_dim, block_size, max_blocks_per_seq, num_blocks,
                                   max_context_len, partition_size, dtype, kv_dtype);
    if (check || num_seqs == 0) return check;
    const bool fp8 = kv_dtype == PKV_FP8_E4M3;
    const int group = num_q_heads / num_kv_heads;
    cudaStream_t s = static_cast<cudaStream_t>(stream);

    const int wcheck = decode_workspace_check(num_seqs, num_q_heads, num_kv_heads, head_dim, block_size,
                                              max_context_len, partition_size, workspace, workspace_bytes);
    if (wcheck) return wcheck;
    const int64_t max_blocks_needed = std::max<int64_t>(1, ceil_div(std::max(max_context_len, 1), block_size));
    int64_t pb = partition_size > 0 ? partition_size / block_size : max_blocks_needed;
    pb = std::min(pb, max_blocks_needed);
    const int64_t parts = ceil_div(max_blocks_needed, pb);
    const size_t need = parts > 1 ? pkv_decode_workspace_size(num_seqs, num_q_heads, head_dim, max_context_len,
                                                              (int)(pb * block_size))
                                  : 0;
    const int64_t grid = (int64_t)num_seqs * parts * num_kv_heads;

    if (checked_mode()) {
        int rc = check_tables(block_tables, context_lens, num_seqs, max_blocks_per_seq, block_size, num_blocks,
                              max_context_len, s);
        if (rc) return rc;
    }

    CUtensorMap tk, tv;
    int rc = make_pool_map(&tk, key_cache, kv_dtype, num_blocks, block_size, num_kv_heads, head_dim);
    if (rc) return rc;
    rc = make_pool_map(&tv, value_cache, kv_dtype, num_blocks, block_size, num_kv_heads, head_dim);
    if (rc) return rc;

    pkv::DecodeParams prm;
    prm.out = out;
    prm.query = query;
    prm.block_tables = block_tables;
    prm.context_lens = context_lens;
    const int64_t rows = (int64_t)num_seqs * num_q_heads * parts;
    const int64_t ml = ((rows * 4 + 15) / 16) * 16;
    prm.ws_max = need ? reinterpret_cast<float*>(workspace) : nullptr;
    prm.ws_sum = need ? reinterpret_cast<float*>(static_cast<char*>(workspace) + ml) : nullptr;
    prm.ws_out = need ? reinterpret_cast<float*>(static_cast<char*>(workspace) + 2 * ml) : nullptr;
    prm.scale_log2 = scale * 1.4426950408889634f * k_scale;
    prm.out_scale = v_scale;
    prm.num_seqs = num_seqs;
    prm.num_q_heads = num_q_heads;
    prm.num_kv_heads = num_kv_heads;
    prm.max_blocks_per_seq = max_blocks_per_seq;
    prm.num_blocks = num_blocks;
    prm.partition_blocks = (int)pb;
    prm.num_partitions = (int)parts;

    const Launch ln{s, pdl};
    if (fp8) {
        rc = dtype == PKV_F16 ? decode_fp8_by_block<__half>(block_size, group, prm, tk, tv, (int)grid, ln)
                              : decode_fp8_by_block<__nv_bfloat16>(block_size, group, prm, tk, tv, (int)grid, ln);
    } else {
        switch (dtype) {
            case PKV_F32: rc = decode_by_dim<float>(head_dim, block_size, group, prm, tk, tv, (int)grid, ln); break;
            case PKV_F16: rc = decode_by_dim<__half>(head_dim, block_size, group, prm, tk, tv, (int)grid, ln); break;
            default:
                rc = decode_by_dim<__nv_bfloat16>(head_dim, block_size, group, prm, tk, tv, (int)grid, ln);
                break;
        }
    }
    if (rc || parts <= 1) return rc;

    pkv::MergeParams mp;
    mp.out = out;
    mp.context_lens = context_lens;
    mp.ws_max = prm.ws_max;
    mp.ws_sum = prm.ws_sum;
    mp.ws_out = prm.ws_out;
    mp.num_seqs = num_seqs;
    mp.num_q_heads = num_q_heads;
    mp.block_size = block_size;
    mp.max_blocks_per_seq = max_blocks_per_seq;
    mp.partition_blocks = (int)pb;
    mp.num_partitions = (int)parts;
    switch (dtype) {
        case PKV_F32: return launch_merge<float>(head_dim, mp, s);
        case PKV_F16: return launch_merge<__half>(head_dim, mp, s);
        default: return launch_merge<__nv_bfloat16>(head_dim, mp, s);
    }
}

}  // namespace

// ============================================================ C ABI
extern "C" {

const char* pkv_status_string(int status) {
    switch (status) {
        case PKV_OK: return "ok";
        case PKV_EINVAL: return "invalid argument";
        case PKV_EUNSUPPORTED: return "unsupported shape or dtype";
        case PKV_ERANGE: return "table entry out of range";
        case PKV_ECUDA: return "CUDA error";
        case PKV_EWORKSPACE: return "workspace missing or too small";
        default: return "unknown status";
    }
}

const char* pkv_last_cuda_error(void) { return g_last_cuda_error; }

int pkv_reshape_and_cache(const void* key, const void* value, void* key_cache, void* value_cache,
                          const int64_t* slot_mapping, int64_t num_tokens, int num_kv_heads, int head_dim,
                          int block_size, int64_t num_blocks, int dtype, pkv_stream_t stream) {
    const int check = reshape_check(key, value, key_cache, value_cache, slot_mapping, num_tokens, num_kv_heads,
                                    head_dim, block_size, num_blocks, dtype, false);
    if (check || num_tokens == 0) return check;
    const int64_t row_bytes = (int64_t)num_kv_heads * head_dim * elem_bytes(dtype);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int64_t num_slots = num_blocks * block_size;
    if (checked_mode()) {
        std::vector<int64_t> sm;
        int rc = fetch(sm, slot_mapping, (size_t)num_tokens, s);
        if (rc) return rc;
        for (int64_t v : sm)
            if (v >= num_slots) return PKV_ERANGE;
    }
    const int row_vecs = (int)(row_bytes / 16);
    const dim3 grid((unsigned)ceil_div(row_vecs, 128), (unsigned)std::min<int64_t>(num_tokens, 65535));
    pkv::reshape_and_cache_kernel<<<grid, 128, 0, s>>>(
        static_cast<const uint4*>(key), static_cast<const uint4*>(value), static_cast<uint4*>(key_cache),
        static_cast<uint4*>(value_cache), slot_mapping, num_tokens, row_vecs, num_slots);
    PKV_CUDA(cudaGetLastError());
    return PKV_OK;
}

int pkv_reshape_and_cache_fp8(const void* key, const void* value, void* key_cache, void* value_cache,
                              const int64_t* slot_mapping, int64_t num_tokens, int num_kv_heads, int head_dim,
                              int block_size, int64_t num_blocks, int src_dtype, float k_scale, float v_scale,
                              pkv_stream_t stream) {
    if (!query_type(src_dtype)) return PKV_EUNSUPPORTED;
    if (num_tokens < 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 || num_blocks <= 0)
        return PKV_EINVAL;
    if (!(std::isfinite(k_scale) && k_scale > 0.f && std::isfinite(v_scale) && v_scale > 0.f)) return PKV_EINVAL;
    const int check = reshape_fp8_check(key, value, key_cache, value_cache, slot_mapping, num_tokens, num_kv_heads,
                                        head_dim, block_size, num_blocks, src_dtype);
    if (check || num_tokens == 0) return check;
    const int64_t row_elems = (int64_t)num_kv_heads * head_dim;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int64_t num_slots = num_blocks * block_size;
    if (checked_mode()) {
        std::vector<int64_t> sm;
        int rc = fetch(sm, slot_mapping, (size_t)num_tokens, s);
        if (rc) return rc;
        for (int64_t v : sm)
            if (v >= num_slots) return PKV_ERANGE;
    }
    const dim3 grid((unsigned)ceil_div(row_elems / 8, 128), (unsigned)std::min<int64_t>(num_tokens, 65535));
    uint2* kc = static_cast<uint2*>(key_cache);
    uint2* vc = static_cast<uint2*>(value_cache);
    switch (src_dtype) {
        case PKV_F32:
            pkv::reshape_and_cache_fp8_kernel<float><<<grid, 128, 0, s>>>(
                static_cast<const float*>(key), static_cast<const float*>(value), kc, vc, slot_mapping, num_tokens,
                (int)row_elems, num_slots, k_scale, v_scale);
            break;
        case PKV_F16:
            pkv::reshape_and_cache_fp8_kernel<__half><<<grid, 128, 0, s>>>(
                static_cast<const __half*>(key), static_cast<const __half*>(value), kc, vc, slot_mapping, num_tokens,
                (int)row_elems, num_slots, k_scale, v_scale);
            break;
        default:
            pkv::reshape_and_cache_fp8_kernel<__nv_bfloat16><<<grid, 128, 0, s>>>(
                static_cast<const __nv_bfloat16*>(key), static_cast<const __nv_bfloat16*>(value), kc, vc, slot_mapping,
                num_tokens, (int)row_elems, num_slots, k_scale, v_scale);
            break;
    }
    PKV_CUDA(cudaGetLastError());
    return PKV_OK;
}

int pkv_copy_blocks(void* const* key_caches, void* const* value_caches, int num_layers,
                    const int64_t* src_dst_pairs, int64_t num_pairs, int64_t block_bytes, int64_t num_blocks,
                    pkv_stream_t stream) {
    if (num_layers < 0 || num_pairs < 0 || block_bytes <= 0 || num_blocks <= 0) return PKV_EINVAL;
    if (block_bytes % 16 != 0) return PKV_EUNSUPPORTED;
    if (num_layers == 0 || num_pairs == 0) return PKV_OK;
    if (!key_caches || !value_caches || !src_dst_pairs || (reinterpret_cast<uintptr_t>(src_dst_pairs) & 7))
        return PKV_EINVAL;
    for (int l = 0; l < num_layers; ++l)
        if (!key_caches[l] || !value_caches[l] || !aligned16(key_caches[l]) || !aligned16(value_caches[l]))
            return PKV_EINVAL;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (checked_mode()) {
        std::vector<int64_t> pr;
        int rc = fetch(pr, src_dst_pairs, (size_t)num_pairs * 2, s);
        if (rc) return rc;
        std::set<int64_t> srcs, dsts;
        for (int64_t i = 0; i < num_pairs; ++i) {
            const int64_t a = pr[2 * i], b = pr[2 * i + 1];
            if (a < 0 || a >= num_blocks || b < 0 || b >= num_blocks) return PKV_ERANGE;
            if (!dsts.insert(b).second) return PKV_ERANGE;
            srcs.insert(a);
        }
        for (int64_t d : dsts)
            if (srcs.count(d)) return PKV_ERANGE;
    }
    const int64_t block_vecs = block_bytes / 16;
    const int64_t per_cta = (int64_t)pkv::kCopyThreads * pkv::kCopyUnroll;
    const unsigned gx = (unsigned)ceil_div(block_vecs, per_cta);
    const unsigned gy = (unsigned)std::min<int64_t>(num_pairs, 65535);
    for (int l0 = 0; l0 < num_layers; l0 += pkv::kMaxLayersPerLaunch) {
        const int nl = std::min(pkv::kMaxLayersPerLaunch, num_layers - l0);
        pkv::LayerPools pools;
        memset(&pools, 0, sizeof pools);
        for (int l = 0; l < nl; ++l) {
            pools.k[l] = static_cast<uint4*>(key_caches[l0 + l]);
            pools.v[l] = static_cast<uint4*>(value_caches[l0 + l]);
        }
        dim3 grid(gx, gy, 2 * nl);
        pkv::copy_blocks_kernel<<<grid, pkv::kCopyThreads, 0, s>>>(pools, src_dst_pairs, num_pairs, block_vecs,
                                                                    num_blocks);
        PKV_CUDA(cudaGetLastError());
    }
    return PKV_OK;
}

int pkv_swap_blocks(const void* src_key_pool, const void* src_value_pool, void* dst_key_pool, void* dst_value_pool,
                    const int64_t* src_dst_pairs, int64_t num_pairs, int64_t block_bytes, int64_t src_num_blocks,
                    int64_t dst_num_blocks, pkv_stream_t stream) {
    if (num_pairs < 0 || block_bytes <= 0 || src_num_blocks <= 0 || dst_num_blocks <= 0) return PKV_EINVAL;
    if (block_bytes % 16 != 0) return PKV_EUNSUPPORTED;
    if (num_pairs == 0) return PKV_OK;
    const void* ptrs[5] = {src_key_pool, src_value_pool, dst_key_pool, dst_value_pool, src_dst_pairs};
    for (const void* q : ptrs) {
        if (!q || (q != src_dst_pairs && !aligned16(q))) return PKV_EINVAL;
        // every buffer must be reachable by the GPU: device, managed or page-locked host memory
        cudaPointerAttributes a;
        if (cudaPointerGetAttributes(&a, q) != cudaSuccess) {
            cudaGetLastError();
            return PKV_EINVAL;
        }
        if (a.type == cudaMemoryTypeUnregistered) return PKV_EINVAL;
    }
    if (reinterpret_cast<uintptr_t>(src_dst_pairs) & 7) return PKV_EINVAL;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int64_t block_vecs = block_bytes / 16;
    const int64_t per_cta = (int64_t)pkv::kCopyThreads * pkv::kCopyUnroll;
    dim3 grid((unsigned)ceil_div(block_vecs, per_cta), (unsigned)std::min<int64_t>(num_pairs, 65535), 2);
    pkv::swap_blocks_kernel<<<grid, pkv::kCopyThreads, 0, s>>>(
        static_cast<const uint4*>(src_key_pool), static_cast<const uint4*>(src_value_pool),
        static_cast<uint4*>(dst_key_pool), static_cast<uint4*>(dst_value_pool), src_dst_pairs, num_pairs, block_vecs,
        src_num_blocks, dst_num_blocks);
    PKV_CUDA(cudaGetLastError());
    return PKV_OK;
}

size_t pkv_decode_workspace_size(int num_seqs, int num_q_heads, int head_dim, int max_context_len,
                                 int partition_size) {
    if (num_seqs <= 0 || num_q_heads <= 0 || head_dim <= 0 || partition_size <= 0 || max_context_len <= 0)
        return 0;
    const int64_t parts = ceil_div(max_context_len, partition_size);
    if (parts <= 1) return 0;
    const int64_t rows = (int64_t)num_seqs * num_q_heads * parts;
    // max and sum (rounded up to 16 bytes each), then the partial outputs
    const int64_t ml = ((rows * 4 + 15) / 16) * 16;
    return (size_t)(2 * ml + rows * head_dim * 4);
}

int pkv_decode_partition_size(int num_seqs, int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                              int max_context_len, int64_t total_context_tokens, int dtype) {
    if (num_seqs < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || num_q_heads % num_kv_heads || head_dim <= 0 ||
        block_size <= 0 || max_context_len < 0 || total_context_tokens < 0 || !elem_bytes(dtype))
        return PKV_EINVAL;
    (void)head_dim;
    const int64_t pairs = (int64_t)num_seqs * num_kv_heads;
    if (max_context_len <= 0 || pairs == 0) return 0;
    // A partition holds at most kMaxPartitionBlocks blocks; a longer context
    // is always split, into equal parts under that cap.
    const int64_t cap = kMaxPartitionBlocks * block_size;
    const int64_t longest = ceil_div(max_context_len, ceil_div(max_context_len, cap));
    auto round_ps = [&](int64_t ps) -> int {
        ps = std::max<int64_t>(ps, 256);
        ps = ceil_div(ps, block_size) * block_size;
        ps = std::min(ps, ceil_div(longest, block_size) * block_size);
        return ps >= max_context_len ? 0 : (int)ps;
    };
    const int64_t target = 4 * (int64_t)sm_count();
    if (pairs * 2 < target) {
        // Small batch: cut contexts so that about four CTAs per SM exist.
        return round_ps(ceil_div(max_context_len, ceil_div(target, pairs)));
    }
    // Enough (sequence, KV head) pairs for every SM: splitting only adds CTA
    // start-up, partial writes and a merge launch -- unless a few contexts are
    // much longer than the rest, whose CTAs would then finish last.  With the
    // total known, contexts beyond 2.5x the mean are cut at 1.5x the mean
    // (measured on B200: lognormal lengths gain ~7%, uniform ones lose ~5-7%
    // when split).
    if (total_context_tokens > 0) {
        const double mean = (double)total_context_tokens / num_seqs;
        if (max_context_len > 2.5 * mean) return round_ps((int64_t)std::ceil(1.5 * mean));
        // E4M3 pools without grouping (one query head per KV head): a CTA
        // streams half the bytes of a 16-bit one and resident CTAs turn over
        // twice as fast, so a batch of fewer than ~22 CTAs per SM ends in a
        // ragged last wave.  Cutting contexts into parts of
        // Hkv * total / (22 * SMs - pairs / 2) tokens (each pair adds half a
        // part on average) makes about 22 CTAs per SM; the merge costs D * 8
        // bytes per extra part, under 1 % of a part's K/V at 512 tokens.  Measured on B200 (d 128,
        // block 16, contexts uniform): 64 x 32 pairs over [128, 2048] gain 3 %
        // and 32 x 32 over [1024, 4096] 13 %, while 128 x 32 pairs, and 256 x
        // 8 KV heads with 8 query heads each (whose merge moves 8x the
        // partials), are fastest unsplit.
        const int64_t waves = 22 * (int64_t)sm_count();
        if (dtype == PKV_FP8_E4M3 && num_q_heads == num_kv_heads && pairs < waves) {
            const double per_part = (double)num_kv_heads * total_context_tokens / (double)(waves - pairs / 2);
            return round_ps(std::max<int64_t>((int64_t)std::ceil(per_part), 512));
        }
    }
    return round_ps(longest);  // 0 unless the longest context exceeds the cap
}

int pkv_paged_attention_decode(void* out, const void* query, const void* key_cache, const void* value_cache,
                               const int32_t* block_tables, const int32_t* context_lens, float scale, int num_seqs,
                               int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                               int max_blocks_per_seq, int64_t num_blocks, int max_context_len, int partition_size,
                               int dtype, void* workspace, size_t workspace_bytes, pkv_stream_t stream) {
    return decode_impl(out, query, key_cache, value_cache, block_tables, context_lens, scale, num_seqs, num_q_heads,
                       num_kv_heads, head_dim, block_size, max_blocks_per_seq, num_blocks, max_context_len,
                       partition_size, dtype, dtype, 1.f, 1.f, workspace, workspace_bytes, stream);
}

int pkv_paged_attention_decode_fp8(void* out, const void* query, const void* key_cache, const void* value_cache,
                                   const int32_t* block_tables, const int32_t* context_lens, float scale,
                                   float k_scale, float v_scale, int num_seqs, int num_q_heads, int num_kv_heads,
                                   int head_dim, int block_size, int max_blocks_per_seq, int64_t num_blocks,
                                   int max_context_len, int partition_size, int dtype, void* workspace,
                                   size_t workspace_bytes, pkv_stream_t stream) {
    if (!(std::isfinite(k_scale) && k_scale > 0.f && std::isfinite(v_scale) && v_scale > 0.f)) return PKV_EINVAL;
    return decode_impl(out, query, key_cache, value_cache, block_tables, context_lens, scale, num_seqs, num_q_heads,
                       num_kv_heads, head_dim, block_size, max_blocks_per_seq, num_blocks, max_context_len,
                       partition_size, dtype, PKV_FP8_E4M3, k_scale, v_scale, workspace, workspace_bytes, stream);
}

int pkv_paged_attention_decode_step(const void* new_keys, const void* new_values, const int64_t* slot_mapping,
                                    int64_t num_new_tokens, void* out, const void* query, void* key_cache,
                                    void* value_cache, const int32_t* block_tables, const int32_t* context_lens,
                                    float scale, int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                                    int block_size, int max_blocks_per_seq, int64_t num_blocks, int max_context_len,
                                    int partition_size, int dtype, void* workspace, size_t workspace_bytes,
                                    pkv_stream_t stream) {
    // Every check of both calls before the first launch, so that a refused
    // step has changed nothing.
    int rc = decode_check(out, query, key_cache, value_cache, block_tables, context_lens, scale, num_seqs,
                          num_q_heads, num_kv_heads, head_dim, block_size, max_blocks_per_seq, num_blocks,
                          max_context_len, partition_size, dtype, dtype);
    if (rc) return rc;
    rc = decode_workspace_check(num_seqs, num_q_heads, num_kv_heads, head_dim, block_size, max_context_len,
                                partition_size, workspace, workspace_bytes);
    if (rc) return rc;
    rc = reshape_check(new_keys, new_values, key_cache, value_cache, slot_mapping, num_new_tokens, num_kv_heads,
                       head_dim, block_size, num_blocks, dtype, false);
    if (rc) return rc;
    rc = pkv_reshape_and_cache(new_keys, new_values, key_cache, value_cache, slot_mapping, num_new_tokens,
                               num_kv_heads, head_dim, block_size, num_blocks, dtype, stream);
    if (rc) return rc;
    return decode_impl(out, query, key_cache, value_cache, block_tables, context_lens, scale, num_seqs, num_q_heads,
                       num_kv_heads, head_dim, block_size, max_blocks_per_seq, num_blocks, max_context_len,
                       partition_size, dtype, dtype, 1.f, 1.f, workspace, workspace_bytes, stream,
                       /*pdl=*/num_new_tokens > 0);
}

int pkv_paged_attention_decode_step_fp8(const void* new_keys, const void* new_values, const int64_t* slot_mapping,
                                        int64_t num_new_tokens, void* out, const void* query, void* key_cache,
                                        void* value_cache, const int32_t* block_tables, const int32_t* context_lens,
                                        float scale, float k_scale, float v_scale, int num_seqs, int num_q_heads,
                                        int num_kv_heads, int head_dim, int block_size, int max_blocks_per_seq,
                                        int64_t num_blocks, int max_context_len, int partition_size, int dtype,
                                        void* workspace, size_t workspace_bytes, pkv_stream_t stream) {
    if (!(std::isfinite(k_scale) && k_scale > 0.f && std::isfinite(v_scale) && v_scale > 0.f)) return PKV_EINVAL;
    int rc = decode_check(out, query, key_cache, value_cache, block_tables, context_lens, scale, num_seqs,
                          num_q_heads, num_kv_heads, head_dim, block_size, max_blocks_per_seq, num_blocks,
                          max_context_len, partition_size, dtype, PKV_FP8_E4M3);
    if (rc) return rc;
    rc = decode_workspace_check(num_seqs, num_q_heads, num_kv_heads, head_dim, block_size, max_context_len,
                                partition_size, workspace, workspace_bytes);
    if (rc) return rc;
    rc = reshape_fp8_check(new_keys, new_values, key_cache, value_cache, slot_mapping, num_new_tokens, num_kv_heads,
                           head_dim, block_size, num_blocks, dtype);
    if (rc) return rc;
    rc = pkv_reshape_and_cache_fp8(new_keys, new_values, key_cache, value_cache, slot_mapping, num_new_tokens,
                                   num_kv_heads, head_dim, block_size, num_blocks, dtype, k_scale, v_scale, stream);
    if (rc) return rc;
    return decode_impl(out, query, key_cache, value_cache, block_tables, context_lens, scale, num_seqs, num_q_heads,
                       num_kv_heads, head_dim, block_size, max_blocks_per_seq, num_blocks, max_context_len,
                       partition_size, dtype, PKV_FP8_E4M3, k_scale, v_scale, workspace, workspace_bytes, stream,
                       /*pdl=*/num_new_tokens > 0);
}

int pkv_set_wait_limit_ns(uint64_t limit_ns) {
    PKV_CUDA(cudaDeviceSynchronize());
    PKV_CUDA(cudaMemcpyToSymbol(pkv::c_main_wait_limit_ns, &limit_ns, sizeof limit_ns));
    PKV_CUDA(cudaDeviceSynchronize());
    return PKV_OK;
}

int pkv_paged_attention_prefill_chunk(void* out, const void* query, const void* key_cache, const void* value_cache,
                                      const int32_t* block_tables, const int32_t* seq_lens,
                                      const int32_t* query_start_loc, int num_chunks, int64_t total_q_tokens,
                                      int max_q_len, float scale, int num_q_heads, int num_kv_heads, int head_dim,
                                      int block_size, int max_blocks_per_seq, int64_t num_blocks, int dtype,
                                      pkv_stream_t stream) {
    if (dtype != PKV_F16 && dtype != PKV_BF16) return elem_bytes(dtype) ? PKV_EUNSUPPORTED : PKV_EUNSUPPORTED;
    if (num_chunks < 0 || total_q_tokens < 0 || max_q_len < 0 || num_q_heads <= 0 || num_kv_heads <= 0 ||
        max_blocks_per_seq <= 0 || num_blocks <= 0 || !std::isfinite(scale))
        return PKV_EINVAL;
    if (num_q_heads % num_kv_heads) return PKV_EINVAL;
    const int group = num_q_heads / num_kv_heads;
    if (!supported_group(group) || (head_dim != 64 && head_dim != 128) ||
        (block_size != 8 && block_size != 16 && block_size != 32))
        return PKV_EUNSUPPORTED;
    if (num_blocks >= (int64_t)INT32_MAX || (int64_t)max_blocks_per_seq * block_size > INT32_MAX ||
        total_q_tokens > INT32_MAX)
        return PKV_EINVAL;
    if (num_chunks == 0 || total_q_tokens == 0 || max_q_len == 0) return PKV_OK;
    if (!out || !query || !key_cache || !value_cache || !block_tables || !seq_lens || !query_start_loc)
        return PKV_EINVAL;
    if (!aligned16(out) || !aligned16(query) || !aligned16(key_cache) || !aligned16(value_cache) ||
        (reinterpret_cast<uintptr_t>(block_tables) & 3) || (reinterpret_cast<uintptr_t>(seq_lens) & 3) ||
        (reinterpret_cast<uintptr_t>(query_start_loc) & 3))
        return PKV_EINVAL;
    cudaStream_t s = static_cast<cudaStream_t>(stream);

    if (checked_mode()) {
        std::vector<int32_t> qsl, lens;
        int rc = fetch(qsl, query_start_loc, (size_t)num_chunks + 1, s);
        if (rc) return rc;
        rc = fetch(lens, seq_lens, (size_t)num_chunks, s);
        if (rc) return rc;
        if (qsl[0] < 0 || qsl[num_chunks] > total_q_tokens) return PKV_ERANGE;
        for (int r = 0; r < num_chunks; ++r) {
            const int n = qsl[r + 1] - qsl[r];
            if (n < 0 || n > max_q_len || lens[r] < n) return PKV_ERANGE;
        }
        rc = check_tables(block_tables, seq_lens, num_chunks, max_blocks_per_seq, block_size, num_blocks,
                          (int64_t)max_blocks_per_seq * block_size, s);
        if (rc) return rc;
    }

    CUtensorMap tq, tk, tv;
    int rc = make_query_map(&tq, query, dtype, total_q_tokens, num_q_heads, head_dim, group);
    if (rc) return rc;
    rc = make_pool_map(&tk, key_cache, dtype, num_blocks, block_size, num_kv_heads, head_dim);
    if (rc) return rc;
    rc = make_pool_map(&tv, value_cache, dtype, num_blocks, block_size, num_kv_heads, head_dim);
    if (rc) return rc;

    const int tile_tokens = 128 / group;
    const int64_t tile_pairs = ceil_div(ceil_div(max_q_len, tile_tokens), 2);
    const int64_t grid = (int64_t)num_chunks * tile_pairs * num_kv_heads;
    if (grid > INT32_MAX) return PKV_EUNSUPPORTED;

    pkv::PrefillParams prm;
    prm.out = out;
    prm.block_tables = block_tables;
    prm.seq_lens = seq_lens;
    prm.query_start_loc = query_start_loc;
    prm.scale_log2 = scale * 1.4426950408889634f;
    prm.num_chunks = num_chunks;
    prm.num_q_heads = num_q_heads;
    prm.num_kv_heads = num_kv_heads;
    prm.max_blocks_per_seq = max_blocks_per_seq;
    prm.block_size = block_size;
    prm.num_blocks = num_blocks;
    prm.tile_pairs = (int)tile_pairs;
    prm.out_scale = 1.f;
    const bool bf16 = dtype == PKV_BF16;
    if (head_dim == 64)
        return bf16 ? prefill_by_group<__nv_bfloat16, 64>(group, prm, tq, tk, tv, (int)grid, s)
                    : prefill_by_group<__half, 64>(group, prm, tq, tk, tv, (int)grid, s);
    return bf16 ? prefill_by_group<__nv_bfloat16, 128>(group, prm, tq, tk, tv, (int)grid, s)
                : prefill_by_group<__half, 128>(group, prm, tq, tk, tv, (int)grid, s);
}

}  // extern "C"

namespace {

// The multi-token decode: every host check, then (unless check_only) the
// launches; pdl launches the attention grid as the programmatic dependent of
// the kernel before it on the stream (this library's append, in the step call).
int decode_multi_impl(void* out, const void* query, const void* key_cache, const void* value_cache,
                      const int32_t* block_tables, const int32_t* seq_lens, const int32_t* query_start_loc,
                      int num_chunks, int64_t total_q_tokens, int max_q_len, int max_seq_len, float scale,
                      int num_q_heads, int num_kv_heads, int head_dim, int block_size, int max_blocks_per_seq,
                      int64_t num_blocks, int partition_size, int dtype, void* workspace, size_t workspace_bytes,
                      pkv_stream_t stream, bool check_only, bool pdl) {
    if (dtype != PKV_F16 && dtype != PKV_BF16) return PKV_EUNSUPPORTED;
    if (num_chunks < 0 || total_q_tokens < 0 || max_q_len < 0 || max_seq_len < 0 || num_q_heads <= 0 ||
        num_kv_heads <= 0 || max_blocks_per_seq <= 0 || num_blocks <= 0 || partition_size < 0 ||
        !std::isfinite(scale))
        return PKV_EINVAL;
    if (num_q_heads % num_kv_heads) return PKV_EINVAL;
    const int group = num_q_heads / num_kv_heads;
    if (!supported_group(group) || (head_dim != 64 && head_dim != 128) ||
        (block_size != 8 && block_size != 16 && block_size != 32))
        return PKV_EUNSUPPORTED;
    if ((int64_t)max_q_len * group > 32) return PKV_EUNSUPPORTED;  // at most two 16-row groups per KV head
    if (partition_size % block_size) return PKV_EINVAL;
    if (num_blocks >= (int64_t)INT32_MAX || (int64_t)max_blocks_per_seq * block_size > INT32_MAX ||
        total_q_tokens > INT32_MAX)
        return PKV_EINVAL;
    if (num_chunks == 0 || total_q_tokens == 0 || max_q_len == 0) return PKV_OK;
    if (!out || !query || !key_cache || !value_cache || !block_tables || !seq_lens || !query_start_loc)
        return PKV_EINVAL;
    if (!aligned16(out) || !aligned16(query) || !aligned16(key_cache) || !aligned16(value_cache) ||
        (reinterpret_cast<uintptr_t>(block_tables) & 3) || (reinterpret_cast<uintptr_t>(seq_lens) & 3) ||
        (reinterpret_cast<uintptr_t>(query_start_loc) & 3))
        return PKV_EINVAL;
    cudaStream_t s = static_cast<cudaStream_t>(stream);

    const int64_t max_blocks_needed = std::max<int64_t>(1, ceil_div(std::max(max_seq_len, 1), block_size));
    int64_t pb = partition_size > 0 ? partition_size / block_size : max_blocks_needed;
    pb = std::min(pb, max_blocks_needed);
    const int64_t parts = ceil_div(max_blocks_needed, pb);
    if (pb > kMaxPartitionBlocks) return PKV_EUNSUPPORTED;
    const size_t need = parts > 1 ? pkv_decode_workspace_size((int)total_q_tokens, num_q_heads, head_dim,
                                                              max_seq_len, (int)(pb * block_size))
                                  : 0;
    if (need > 0 && (!workspace || workspace_bytes < need || !aligned16(workspace))) return PKV_EWORKSPACE;
    const int64_t items = (int64_t)num_chunks * parts * num_kv_heads;  // (chunk, partition, KV head)
    if (items >= (int64_t(1) << 30)) return PKV_EUNSUPPORTED;  // the kernel ranks items in 32 bits

    if (checked_mode()) {
        std::vector<int32_t> qsl, lens;
        int rc = fetch(qsl, query_start_loc, (size_t)num_chunks + 1, s);
        if (rc) return rc;
        rc = fetch(lens, seq_lens, (size_t)num_chunks, s);
        if (rc) return rc;
        if (qsl[0] < 0 || qsl[num_chunks] > total_q_tokens) return PKV_ERANGE;
        for (int r = 0; r < num_chunks; ++r) {
            const int n = qsl[r + 1] - qsl[r];
            if (n < 0 || n > max_q_len || lens[r] < n) return PKV_ERANGE;
        }
        rc = check_tables(block_tables, seq_lens, num_chunks, max_blocks_per_seq, block_size, num_blocks,
                          max_seq_len, s);
        if (rc) return rc;
    }
    if (check_only) return PKV_OK;

    CUtensorMap tq, tk, tv;
    // Q: 32 / G tokens x G heads = the 32 rows of a KV head; K/V: one box per block
    int rc = make_query_map(&tq, query, dtype, total_q_tokens, num_q_heads, head_dim, group, 32 / group);
    if (rc) return rc;
    rc = make_pool_map(&tk, key_cache, dtype, num_blocks, block_size, num_kv_heads, head_dim);
    if (rc) return rc;
    rc = make_pool_map(&tv, value_cache, dtype, num_blocks, block_size, num_kv_heads, head_dim);
    if (rc) return rc;

    pkv::MultiParams prm;
    prm.out = out;
    prm.block_tables = block_tables;
    prm.seq_lens = seq_lens;
    prm.query_start_loc = query_start_loc;
    const int64_t rows = total_q_tokens * num_q_heads * parts;
    const int64_t ml = ((rows * 4 + 15) / 16) * 16;
    prm.ws_max = need ? reinterpret_cast<float*>(workspace) : nullptr;
    prm.ws_sum = need ? reinterpret_cast<float*>(static_cast<char*>(workspace) + ml) : nullptr;
    prm.ws_out = need ? reinterpret_cast<float*>(static_cast<char*>(workspace) + 2 * ml) : nullptr;
    prm.scale_log2 = scale * 1.4426950408889634f;
    prm.num_chunks = num_chunks;
    prm.num_q_heads = num_q_heads;
    prm.num_kv_heads = num_kv_heads;
    prm.group = group;
    prm.block_size = block_size;
    prm.max_blocks_per_seq = max_blocks_per_seq;
    prm.num_blocks = num_blocks;
    prm.partition_blocks = (int)pb;
    prm.num_partitions = (int)parts;
    prm.total_q_tokens = total_q_tokens;
    const int lpt = num_chunks <= pkv::kMultiLptChunks ? 1 : 0;
    const bool bf16 = dtype == PKV_BF16;
    const Launch la{s, pdl};
    if (head_dim == 64)
        rc = bf16 ? launch_multi<__nv_bfloat16, 64>(prm, lpt, tq, tk, tv, items, la)
                  : launch_multi<__half, 64>(prm, lpt, tq, tk, tv, items, la);
    else
        rc = bf16 ? launch_multi<__nv_bfloat16, 128>(prm, lpt, tq, tk, tv, items, la)
                  : launch_multi<__half, 128>(prm, lpt, tq, tk, tv, items, la);
    if (rc || parts <= 1) return rc;

    pkv::MultiMergeParams mp;
    mp.out = out;
    mp.seq_lens = seq_lens;
    mp.query_start_loc = query_start_loc;
    mp.ws_max = prm.ws_max;
    mp.ws_sum = prm.ws_sum;
    mp.ws_out = prm.ws_out;
    mp.num_chunks = num_chunks;
    mp.num_q_heads = num_q_heads;
    mp.total_q_tokens = total_q_tokens;
    mp.block_size = block_size;
    mp.max_blocks_per_seq = max_blocks_per_seq;
    mp.partition_blocks = (int)pb;
    mp.num_partitions = (int)parts;
    const int64_t warps = total_q_tokens * num_q_heads;
    const dim3 mgrid((unsigned)ceil_div(warps, 4));
    const Launch ln{s, true};  // follows this library's own attention kernel (see launch_merge)
    if (head_dim == 64)
        return bf16 ? launch_kernel(pkv::paged_decode_multi_merge_kernel<__nv_bfloat16, 64>, mgrid, dim3(128), 0, ln, mp)
                    : launch_kernel(pkv::paged_decode_multi_merge_kernel<__half, 64>, mgrid, dim3(128), 0, ln, mp);
    return bf16 ? launch_kernel(pkv::paged_decode_multi_merge_kernel<__nv_bfloat16, 128>, mgrid, dim3(128), 0, ln, mp)
                : launch_kernel(pkv::paged_decode_multi_merge_kernel<__half, 128>, mgrid, dim3(128), 0, ln, mp);
}

}  // namespace

extern "C" {

int pkv_paged_attention_decode_multi(void* out, const void* query, const void* key_cache, const void* value_cache,
                                     const int32_t* block_tables, const int32_t* seq_lens,
                                     const int32_t* query_start_loc, int num_chunks, int64_t total_q_tokens,
                                     int max_q_len, int max_seq_len, float scale, int num_q_heads, int num_kv_heads,
                                     int head_dim, int block_size, int max_blocks_per_seq, int64_t num_blocks,
                                     int partition_size, int dtype, void* workspace, size_t workspace_bytes,
                                     pkv_stream_t stream) {
    return decode_multi_impl(out, query, key_cache, value_cache, block_tables, seq_lens, query_start_loc, num_chunks,
                             total_q_tokens, max_q_len, max_seq_len, scale, num_q_heads, num_kv_heads, head_dim,
                             block_size, max_blocks_per_seq, num_blocks, partition_size, dtype, workspace,
                             workspace_bytes, stream, false, false);
}

int pkv_paged_attention_decode_multi_step(const void* new_keys, const void* new_values, const int64_t* slot_mapping,
                                          int64_t num_new_tokens, void* out, const void* query, void* key_cache,
                                          void* value_cache, const int32_t* block_tables, const int32_t* seq_lens,
                                          const int32_t* query_start_loc, int num_chunks, int64_t total_q_tokens,
                                          int max_q_len, int max_seq_len, float scale, int num_q_heads,
                                          int num_kv_heads, int head_dim, int block_size, int max_blocks_per_seq,
                                          int64_t num_blocks, int partition_size, int dtype, void* workspace,
                                          size_t workspace_bytes, pkv_stream_t stream) {
    // Every check of both calls before the first launch, so that a refused
    // step has changed nothing.
    int rc = decode_multi_impl(out, query, key_cache, value_cache, block_tables, seq_lens, query_start_loc,
                               num_chunks, total_q_tokens, max_q_len, max_seq_len, scale, num_q_heads, num_kv_heads,
                               head_dim, block_size, max_blocks_per_seq, num_blocks, partition_size, dtype, workspace,
                               workspace_bytes, stream, true, false);
    if (rc) return rc;
    rc = reshape_check(new_keys, new_values, key_cache, value_cache, slot_mapping, num_new_tokens, num_kv_heads,
                       head_dim, block_size, num_blocks, dtype, false);
    if (rc) return rc;
    rc = pkv_reshape_and_cache(new_keys, new_values, key_cache, value_cache, slot_mapping, num_new_tokens,
                               num_kv_heads, head_dim, block_size, num_blocks, dtype, stream);
    if (rc) return rc;
    return decode_multi_impl(out, query, key_cache, value_cache, block_tables, seq_lens, query_start_loc, num_chunks,
                             total_q_tokens, max_q_len, max_seq_len, scale, num_q_heads, num_kv_heads, head_dim,
                             block_size, max_blocks_per_seq, num_blocks, partition_size, dtype, workspace,
                             workspace_bytes, stream, false, /*pdl=*/num_new_tokens > 0);
}

int pkv_decode_multi_partition_size(int num_chunks, int num_kv_heads, int block_size, int max_seq_len) {
    if (num_chunks < 0 || num_kv_heads <= 0 || block_size <= 0 || max_seq_len < 0) return PKV_EINVAL;
    const int64_t pairs = (int64_t)num_chunks * num_kv_heads;
    if (max_seq_len <= 0 || pairs == 0) return 0;
    // At least two work items per SM over the whole launch: the persistent
    // CTAs take them longest first, and an item boundary costs about two key
    // tiles, so (chunk, KV head) pairs are split only when there are fewer;
    // partitions of at least 256 tokens, in whole 128-key tiles.  Never more
    // than kMaxPartitionBlocks blocks.
    const int64_t target = 2 * (int64_t)sm_count();
    const int64_t cap = kMaxPartitionBlocks * block_size;
    const int64_t parts = std::max(std::max<int64_t>(1, ceil_div(target, pairs)), ceil_div(max_seq_len, cap));
    int64_t ps = std::max<int64_t>(256, ceil_div(max_seq_len, parts));
    const int64_t unit = 128 % block_size == 0 ? 128 : block_size;
    ps = std::min(ceil_div(ps, unit) * unit, cap);
    return ps >= max_seq_len ? 0 : (int)ps;
}

size_t pkv_prefill_fp8_workspace_size(int num_chunks, int max_blocks_per_seq, int block_size, int num_kv_heads,
                                      int head_dim, int64_t total_q_tokens, int num_q_heads, int dtype) {
    if (num_chunks <= 0 || max_blocks_per_seq <= 0 || block_size <= 0 || num_kv_heads <= 0 || head_dim <= 0 ||
        total_q_tokens < 0 || num_q_heads <= 0)
        return 0;
    auto al = [](int64_t x) { return ((x + 1023) / 1024) * 1024; };
    const int64_t entries = (int64_t)num_chunks * max_blocks_per_seq;
    const int64_t pool = entries * block_size * num_kv_heads * head_dim * 2;
    const int64_t q = dtype == PKV_BF16 ? total_q_tokens * num_q_heads * head_dim * 2 : 0;
    return (size_t)(al(q) + 2 * al(pool) + al(entries * 4));
}

int pkv_paged_attention_prefill_chunk_fp8(void* out, const void* query, const void* key_cache, const void* value_cache,
                                          const int32_t* block_tables, const int32_t* seq_lens,
                                          const int32_t* query_start_loc, int num_chunks, int64_t total_q_tokens,
                                          int max_q_len, float scale, float k_scale, float v_scale, int num_q_heads,
                                          int num_kv_heads, int head_dim, int block_size, int max_blocks_per_seq,
                                          int64_t num_blocks, int dtype, void* workspace, size_t workspace_bytes,
                                          pkv_stream_t stream) {
    if (dtype != PKV_F16 && dtype != PKV_BF16) return PKV_EUNSUPPORTED;
    if (num_chunks < 0 || total_q_tokens < 0 || max_q_len < 0 || num_q_heads <= 0 || num_kv_heads <= 0 ||
        max_blocks_per_seq <= 0 || num_blocks <= 0 || !std::isfinite(scale))
        return PKV_EINVAL;
    if (!(std::isfinite(k_scale) && k_scale > 0.f && std::isfinite(v_scale) && v_scale > 0.f)) return PKV_EINVAL;
    if (num_q_heads % num_kv_heads) return PKV_EINVAL;
    const int group = num_q_heads / num_kv_heads;
    if (!supported_group(group) || (head_dim != 64 && head_dim != 128) ||
        (block_size != 8 && block_size != 16 && block_size != 32))
        return PKV_EUNSUPPORTED;
    const int64_t entries = (int64_t)num_chunks * max_blocks_per_seq;
    if (entries >= (int64_t)INT32_MAX || (int64_t)max_blocks_per_seq * block_size > INT32_MAX ||
        total_q_tokens > INT32_MAX || num_blocks >= (int64_t)INT32_MAX)
        return PKV_EINVAL;
    if (num_chunks == 0 || total_q_tokens == 0 || max_q_len == 0) return PKV_OK;
    if (!out || !query || !key_cache || !value_cache || !block_tables || !seq_lens || !query_start_loc)
        return PKV_EINVAL;
    if (!aligned16(out) || !aligned16(query) || !aligned16(key_cache) || !aligned16(value_cache) ||
        (reinterpret_cast<uintptr_t>(block_tables) & 3) || (reinterpret_cast<uintptr_t>(seq_lens) & 3) ||
        (reinterpret_cast<uintptr_t>(query_start_loc) & 3))
        return PKV_EINVAL;
    const size_t need = pkv_prefill_fp8_workspace_size(num_chunks, max_blocks_per_seq, block_size, num_kv_heads,
                                                       head_dim, total_q_tokens, num_q_heads, dtype);
    if (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255))
        return PKV_EWORKSPACE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (checked_mode()) {
        std::vector<int32_t> qsl, lens;
        int rc = fetch(qsl, query_start_loc, (size_t)num_chunks + 1, s);
        if (rc) return rc;
        rc = fetch(lens, seq_lens, (size_t)num_chunks, s);
        if (rc) return rc;
        if (qsl[0] < 0 || qsl[num_chunks] > total_q_tokens) return PKV_ERANGE;
        for (int r = 0; r < num_chunks; ++r) {
            const int n = qsl[r + 1] - qsl[r];
            if (n < 0 || n > max_q_len || lens[r] < n) return PKV_ERANGE;
        }
        rc = check_tables(block_tables, seq_lens, num_chunks, max_blocks_per_seq, block_size, num_blocks,
                          (int64_t)max_blocks_per_seq * block_size, s);
        if (rc) return rc;
    }
    // workspace: [f16 query (bf16 input only)] [f16 K scratch pool] [f16 V scratch pool] [scratch tables]
    auto al = [](int64_t x) { return ((x + 1023) / 1024) * 1024; };
    const int64_t pool = entries * block_size * num_kv_heads * head_dim * 2;
    const int64_t qbytes = dtype == PKV_BF16 ? total_q_tokens * num_q_heads * head_dim * 2 : 0;
    char* ws = static_cast<char*>(workspace);
    void* q16 = dtype == PKV_BF16 ? (void*)ws : const_cast<void*>(query);
    void* k16 = ws + al(qbytes);
    void* v16 = ws + al(qbytes) + al(pool);
    int32_t* bt16 = reinterpret_cast<int32_t*>(ws + al(qbytes) + 2 * al(pool));
    const int block_vecs = block_size * num_kv_heads * head_dim / 16;  // 16-byte vectors of codes per block
    pkv::widen_fp8_blocks_kernel<<<(unsigned)entries, 256, 0, s>>>(
        static_cast<const uint4*>(key_cache), static_cast<const uint4*>(value_cache), static_cast<uint4*>(k16),
        static_cast<uint4*>(v16), block_tables, seq_lens, bt16, max_blocks_per_seq, block_size, num_blocks,
        block_vecs);
    PKV_CUDA(cudaGetLastError());
    if (dtype == PKV_BF16) {
        const int64_t pairs = total_q_tokens * num_q_heads * head_dim / 2;
        const unsigned g = (unsigned)std::min<int64_t>(ceil_div(pairs, 256), 4 * (int64_t)sm_count());
        pkv::bf16_to_f16_kernel<<<g, 256, 0, s>>>(static_cast<const uint32_t*>(query), static_cast<uint32_t*>(q16),
                                                   pairs);
        PKV_CUDA(cudaGetLastError());
    }

    CUtensorMap tq, tk, tv;
    int rc = make_query_map(&tq, q16, PKV_F16, total_q_tokens, num_q_heads, head_dim, group);
    if (rc) return rc;
    rc = make_pool_map(&tk, k16, PKV_F16, entries, block_size, num_kv_heads, head_dim);
    if (rc) return rc;
    rc = make_pool_map(&tv, v16, PKV_F16, entries, block_size, num_kv_heads, head_dim);
    if (rc) return rc;

    const int tile_tokens = 128 / group;
    const int64_t tile_pairs = ceil_div(ceil_div(max_q_len, tile_tokens), 2);
    const int64_t grid = (int64_t)num_chunks * tile_pairs * num_kv_heads;
    if (grid > INT32_MAX) return PKV_EUNSUPPORTED;
    pkv::PrefillParams prm;
    prm.out = out;
    prm.block_tables = bt16;
    prm.seq_lens = seq_lens;
    prm.query_start_loc = query_start_loc;
    prm.scale_log2 = scale * 1.4426950408889634f * k_scale;
    prm.out_scale = v_scale;
    prm.num_chunks = num_chunks;
    prm.num_q_heads = num_q_heads;
    prm.num_kv_heads = num_kv_heads;
    prm.max_blocks_per_seq = max_blocks_per_seq;
    prm.block_size = block_size;
    prm.num_blocks = entries;
    prm.tile_pairs = (int)tile_pairs;
    const bool bf16 = dtype == PKV_BF16;
    if (head_dim == 64)
        return bf16 ? prefill_by_group<__half, 64, __nv_bfloat16>(group, prm, tq, tk, tv, (int)grid, s)
                    : prefill_by_group<__half, 64>(group, prm, tq, tk, tv, (int)grid, s);
    return bf16 ? prefill_by_group<__half, 128, __nv_bfloat16>(group, prm, tq, tk, tv, (int)grid, s)
                : prefill_by_group<__half, 128>(group, prm, tq, tk, tv, (int)grid, s);
}

int pkv_get_device_error(uint32_t* host_err, pkv_stream_t stream) {
    if (!host_err) return PKV_EINVAL;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    unsigned int v = 0;
    PKV_CUDA(cudaMemcpyFromSymbolAsync(&v, pkv::g_device_error, sizeof v, 0, cudaMemcpyDeviceToHost, s));
    const unsigned int zero = 0;
    PKV_CUDA(cudaMemcpyToSymbolAsync(pkv::g_device_error, &zero, sizeof zero, 0, cudaMemcpyHostToDevice, s));
    PKV_CUDA(cudaStreamSynchronize(s));
    *host_err = v;
    return PKV_OK;
}

}  // extern "C"

// ============================================================ decode without caller-provided scratch
// Some callers cannot allocate device memory when they call decode: code that
// runs inside another framework's allocator-controlled region, plugins that are
// handed only the tensors of one operation, or a serving loop that must not
// touch the allocator between steps.  For them the split-K scratch lives in a
// file-scope device array owned by the library.  The name below is a host-side
// stand-in in host code, so its device address is looked up once per device
// with cudaGetSymbolAddress and passed to the kernels as an ordinary pointer.
static __device__ __align__(256) unsigned char g_static_decode_scratch[PKV_STATIC_DECODE_SCRATCH_BYTES];

namespace {

// Device address of the scratch array in the current device's current
// context, looked up once per context (with that device current) and cached.
// A __device__ array has one address per CUDA context, so the cache is keyed
// by the context, not by the device number: a caller on a context of its own
// (driver API) gets that context's copy.
using CtxGetCurrentFn = CUresult (*)(CUcontext*);

CtxGetCurrentFn ctx_get_current_fn() {
    static CtxGetCurrentFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<CtxGetCurrentFn>(p);
    });
    return fn;
}

void* static_scratch_address(int* rc) {
    static std::mutex mu;
    constexpr int kSlots = 64;
    static CUcontext ctx_of[kSlots] = {};
    static void* addr_of[kSlots] = {};
    CtxGetCurrentFn get_ctx = ctx_get_current_fn();
    CUcontext ctx = nullptr;
    void* looked = nullptr;
    if (!get_ctx || get_ctx(&ctx) != CUDA_SUCCESS) {
        snprintf(g_last_cuda_error, sizeof g_last_cuda_error, "cuCtxGetCurrent unavailable or failed");
        *rc = PKV_ECUDA;
        return nullptr;
    }
    if (!ctx) {
        // No context current on this host thread yet: the runtime's lookup
        // makes the current device's primary context current.
        cudaError_t e = cudaGetSymbolAddress(&looked, g_static_decode_scratch);
        if (e != cudaSuccess || !looked) {
            *rc = cuda_fail(e != cudaSuccess ? e : cudaErrorInvalidSymbol, "cudaGetSymbolAddress(scratch)");
            return nullptr;
        }
        if (get_ctx(&ctx) != CUDA_SUCCESS || !ctx) {
            snprintf(g_last_cuda_error, sizeof g_last_cuda_error, "no current CUDA context");
            *rc = PKV_ECUDA;
            return nullptr;
        }
    }
    std::lock_guard<std::mutex> lock(mu);
    int free_slot = -1;
    for (int i = 0; i < kSlots; ++i) {
        if (ctx_of[i] == ctx) {
            *rc = PKV_OK;
            return addr_of[i];
        }
        if (!ctx_of[i] && free_slot < 0) free_slot = i;
    }
    if (free_slot < 0) {
        *rc = PKV_EUNSUPPORTED;
        return nullptr;
    }
    if (!looked) {
        cudaError_t e = cudaGetSymbolAddress(&looked, g_static_decode_scratch);
        if (e != cudaSuccess || !looked) {
            *rc = cuda_fail(e != cudaSuccess ? e : cudaErrorInvalidSymbol, "cudaGetSymbolAddress(scratch)");
            return nullptr;
        }
    }
    ctx_of[free_slot] = ctx;
    addr_of[free_slot] = looked;
    *rc = PKV_OK;
    return looked;
}

}  // namespace

extern "C" int pkv_paged_attention_decode_static_scratch(
    void* out, const void* query, const void* key_cache, const void* value_cache, const int32_t* block_tables,
    const int32_t* context_lens, float scale, int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
    int block_size, int max_blocks_per_seq, int64_t num_blocks, int max_context_len, int partition_size, int dtype,
    pkv_stream_t stream) {
    // The decode's own argument checks first, so that both entry points return
    // the same status for the same bad input; then the size check: a request
    // that needs more scratch than the array holds is refused before any
    // device work.
    const int check = decode_check(out, query, key_cache, value_cache, block_tables, context_lens, scale, num_seqs,
                                   num_q_heads, num_kv_heads, head_dim, block_size, max_blocks_per_seq, num_blocks,
                                   max_context_len, partition_size, dtype, dtype);
    if (check) return check;
    int64_t ps = partition_size;
    if (ps > 0 && block_size > 0 && max_context_len > 0) {
        const int64_t max_blocks = ceil_div(max_context_len, block_size);
        ps = std::min<int64_t>(ps, max_blocks * block_size);  // the clamp the decode applies
    }
    const size_t need = ps > 0 ? pkv_decode_workspace_size(num_seqs, num_q_heads, head_dim, max_context_len, (int)ps)
                               : 0;
    if (need > (size_t)PKV_STATIC_DECODE_SCRATCH_BYTES) return PKV_EWORKSPACE;
    void* scratch = nullptr;
    if (need > 0) {
        int rc = PKV_OK;
        scratch = static_scratch_address(&rc);
        if (rc) return rc;
    }
    return pkv_paged_attention_decode(out, query, key_cache, value_cache, block_tables, context_lens, scale, num_seqs,
                                      num_q_heads, num_kv_heads, head_dim, block_size, max_blocks_per_seq,
                                      num_blocks, max_context_len, partition_size, dtype, scratch,
                                      need > 0 ? (size_t)PKV_STATIC_DECODE_SCRATCH_BYTES : 0, stream);
}
