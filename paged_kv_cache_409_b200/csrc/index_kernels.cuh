// index_kernels.cuh -- the two indexing kernels of the paged cache:
//   reshape_and_cache (write new tokens' K/V into their physical slots) and
//   copy_blocks (copy-on-write of shared blocks).
// Both are pure data movement in 16-byte vectors, bounded by HBM bandwidth
// (or by launch latency when the token count is small).
#pragma once

#include "ptx.cuh"

namespace pkv {

// Grid (x, y): blockIdx.x picks a 128-vector slice of a row, y strides over
// tokens, so a small batch (one new token per sequence) still spreads over
// hundreds of CTAs with one vector of K and one of V per thread.  A token's K
// row and V row are each contiguous (num_kv_heads * head_dim elements) in the
// source and, in the [num_blocks, block_size, num_kv_heads, head_dim] pool, at
// row `slot`.
__global__ void __launch_bounds__(128) reshape_and_cache_kernel(const uint4* __restrict__ key,
                                                                const uint4* __restrict__ value,
                                                                uint4* __restrict__ key_cache,
                                                                uint4* __restrict__ value_cache,
                                                                const int64_t* __restrict__ slot_mapping,
                                                                int64_t num_tokens, int row_vecs,
                                                                int64_t num_slots) {
    // A decode launched as this grid's programmatic dependent may start its
    // prologue now; it waits for this grid's writes before it reads the pools.
    griddep_launch_dependents();
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    for (int64_t t = blockIdx.y; t < num_tokens; t += gridDim.y) {
        const int64_t slot = slot_mapping[t];
        if (slot < 0) continue;  // padding token
        if (slot >= num_slots) {
            if (i == 0) flag_error(PKV_DEVERR_SLOT);
            continue;
        }
        if (i < row_vecs) {
            const uint4 a = key[t * row_vecs + i];
            const uint4 b = value[t * row_vecs + i];
            key_cache[slot * row_vecs + i] = a;
            value_cache[slot * row_vecs + i] = b;
        }
    }
}

// ---- reshape_and_cache into FP8 (E4M3) pools.
// A stored code is the E4M3 value nearest to x / scale (ties to even,
// saturated at 448).  The quotient is formed in fp32 with rounding to odd --
// the truncated quotient with its last bit set when the division was inexact
// (Boldo and Melquiond, "Emulation of FMA and correctly rounded sums: proved
// algorithms using rounding to odd", 2008) -- so that the one rounding to
// E4M3 that follows gives the nearest value to the EXACT quotient: with 24
// significant bits against E4M3's 4, round-to-odd followed by round-to-nearest
// is a single correct rounding.  NaN is stored as 0x7F.
__device__ __forceinline__ float quotient_round_to_odd(float x, float scale) {
    float q = __fdiv_rz(x, scale);
    if (isfinite(q)) {
        const float r = fmaf(-q, scale, x);  // exact remainder of the truncated quotient
        if (r != 0.f) q = __uint_as_float(__float_as_uint(q) | 1u);
    } else if (isnan(q)) {
        q = __uint_as_float(0x7fc00000u);
    }
    return q;
}

template <typename TS>
__device__ __forceinline__ void load8(const TS* p, float (&f)[8]) {
    if constexpr (sizeof(TS) == 4) {
        const float4 a = reinterpret_cast<const float4*>(p)[0], b = reinterpret_cast<const float4*>(p)[1];
        f[0] = a.x, f[1] = a.y, f[2] = a.z, f[3] = a.w, f[4] = b.x, f[5] = b.y, f[6] = b.z, f[7] = b.w;
    } else {
        Elem<TS>::unpack16(*reinterpret_cast<const uint4*>(p), f);
    }
}

__device__ __forceinline__ uint2 quantise8(const float (&f)[8], float scale) {
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
        w[i] = e4m3x2_from_f32(quotient_round_to_odd(f[2 * i + 1], scale), quotient_round_to_odd(f[2 * i], scale));
    return make_uint2(w[0] | (w[1] << 16), w[2] | (w[3] << 16));
}

// Grid (x, y) as for reshape_and_cache_kernel: blockIdx.x picks 128 groups
// of 8 consecutive elements of a row, y strides over tokens; each thread
// quantises one group of the token's K row and the same group of its V row.
template <typename TS>
__global__ void __launch_bounds__(128) reshape_and_cache_fp8_kernel(const TS* __restrict__ key,
                                                                    const TS* __restrict__ value,
                                                                    uint2* __restrict__ key_cache,
                                                                    uint2* __restrict__ value_cache,
                                                                    const int64_t* __restrict__ slot_mapping,
                                                                    int64_t num_tokens, int row_elems,
                                                                    int64_t num_slots, float k_scale, float v_scale) {
    griddep_launch_dependents();  // as in reshape_and_cache_kernel
    const int groups = row_elems / 8;
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    for (int64_t t = blockIdx.y; t < num_tokens; t += gridDim.y) {
        const int64_t slot = slot_mapping[t];
        if (slot < 0) continue;
        if (slot >= num_slots) {
            if (i == 0) flag_error(PKV_DEVERR_SLOT);
            continue;
        }
        if (i < groups) {
            float kf[8], vf[8];
            load8(key + t * row_elems + 8 * i, kf);
            load8(value + t * row_elems + 8 * i, vf);
            key_cache[slot * groups + i] = quantise8(kf, k_scale);
            value_cache[slot * groups + i] = quantise8(vf, v_scale);
        }
    }
}

// ---- widening of FP8 pools for the chunked prefill.
// One CTA per block-table entry (chunk r, logical block b): the E4M3 codes of
// that physical block's K and V are written as f16 (exact: every E4M3 value is
// an f16 value) to block r * max_blocks + b of two f16 scratch pools, and the
// scratch table entry is that index (-1 for blocks past the sequence or with
// an id outside the pool, which also sets PKV_DEVERR_BLOCK_ID).
__device__ __forceinline__ void widen16(const uint4 x, uint4& lo, uint4& hi) {
    lo.x = f16x2_from_e4m3x2(static_cast<uint16_t>(x.x));
    lo.y = f16x2_from_e4m3x2(static_cast<uint16_t>(x.x >> 16));
    lo.z = f16x2_from_e4m3x2(static_cast<uint16_t>(x.y));
    lo.w = f16x2_from_e4m3x2(static_cast<uint16_t>(x.y >> 16));
    hi.x = f16x2_from_e4m3x2(static_cast<uint16_t>(x.z));
    hi.y = f16x2_from_e4m3x2(static_cast<uint16_t>(x.z >> 16));
    hi.z = f16x2_from_e4m3x2(static_cast<uint16_t>(x.w));
    hi.w = f16x2_from_e4m3x2(static_cast<uint16_t>(x.w >> 16));
}

__global__ void __launch_bounds__(256) widen_fp8_blocks_kernel(const uint4* __restrict__ kc8,
                                                               const uint4* __restrict__ vc8,
                                                               uint4* __restrict__ kc16, uint4* __restrict__ vc16,
                                                               const int32_t* __restrict__ block_tables,
                                                               const int32_t* __restrict__ seq_lens,
                                                               int32_t* __restrict__ tables_out, int max_blocks,
                                                               int block_size, int64_t num_blocks, int block_vecs) {
    const int64_t e = blockIdx.x;
    const int64_t r = e / max_blocks;
    const int b = static_cast<int>(e - r * max_blocks);
    const int len = max(seq_lens[r], 0);
    const int nblk = min((len + block_size - 1) / block_size, max_blocks);
    int id = -1;
    if (b < nblk) {
        id = block_tables[e];
        if (id < 0 || id >= num_blocks) {
            if (threadIdx.x == 0) flag_error(PKV_DEVERR_BLOCK_ID);
            id = -1;
        }
    }
    if (threadIdx.x == 0) tables_out[e] = id >= 0 ? static_cast<int32_t>(e) : -1;
    if (id < 0) return;
    const uint4* ks = kc8 + static_cast<int64_t>(id) * block_vecs;
    const uint4* vs = vc8 + static_cast<int64_t>(id) * block_vecs;
    uint4* kd = kc16 + e * 2 * block_vecs;
    uint4* vd = vc16 + e * 2 * block_vecs;
    for (int i = threadIdx.x; i < block_vecs; i += blockDim.x) {
        const uint4 a = ks[i], c = vs[i];
        uint4 lo, hi;
        widen16(a, lo, hi);
        kd[2 * i] = lo;
        kd[2 * i + 1] = hi;
        widen16(c, lo, hi);
        vd[2 * i] = lo;
        vd[2 * i + 1] = hi;
    }
}

// bf16 -> f16, round to nearest even (grid-stride over pairs).
__global__ void __launch_bounds__(256) bf16_to_f16_kernel(const uint32_t* __restrict__ src, uint32_t* __restrict__ dst,
                                                          int64_t pairs) {
    for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < pairs;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const float2 f = Elem<__nv_bfloat16>::pair(src[i]);
        dst[i] = pack_half2(f.x, f.y);
    }
}

constexpr int kMaxLayersPerLaunch = 32;

struct LayerPools {
    uint4* k[kMaxLayersPerLaunch];
    uint4* v[kMaxLayersPerLaunch];
};

constexpr int kCopyThreads = 256;
constexpr int kCopyUnroll = 4;

// grid.x: chunks of one block (kCopyThreads * kCopyUnroll vectors each),
// grid.y: pairs (grid-stride), grid.z: layer * 2 + (0 = K, 1 = V).
__global__ void __launch_bounds__(kCopyThreads) copy_blocks_kernel(const LayerPools pools,
                                                                   const int64_t* __restrict__ pairs,
                                                                   int64_t num_pairs, int64_t block_vecs,
                                                                   int64_t num_blocks) {
    const int layer = blockIdx.z >> 1;
    uint4* base = (blockIdx.z & 1) ? pools.v[layer] : pools.k[layer];
    const int64_t first = static_cast<int64_t>(blockIdx.x) * kCopyThreads * kCopyUnroll + threadIdx.x;
    for (int64_t p = blockIdx.y; p < num_pairs; p += gridDim.y) {
        const int64_t src = pairs[2 * p];
        const int64_t dst = pairs[2 * p + 1];
        if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) {
            if (threadIdx.x == 0 && blockIdx.x == 0 && blockIdx.z == 0) flag_error(PKV_DEVERR_PAIR);
            continue;
        }
        const uint4* s = base + src * block_vecs;
        uint4* d = base + dst * block_vecs;
        uint4 r[kCopyUnroll];
#pragma unroll
        for (int u = 0; u < kCopyUnroll; ++u) {
            const int64_t i = first + u * kCopyThreads;
            if (i < block_vecs) r[u] = s[i];
        }
#pragma unroll
        for (int u = 0; u < kCopyUnroll; ++u) {
            const int64_t i = first + u * kCopyThreads;
            if (i < block_vecs) d[i] = r[u];
        }
    }
}

// Block moves between two pools (device HBM and/or page-locked host memory,
// reached through unified addressing): grid.x chunks of a block, grid.y pairs
// (grid-stride), grid.z 0 = K, 1 = V.
__global__ void __launch_bounds__(kCopyThreads) swap_blocks_kernel(const uint4* __restrict__ src_k,
                                                                   const uint4* __restrict__ src_v,
                                                                   uint4* __restrict__ dst_k, uint4* __restrict__ dst_v,
                                                                   const int64_t* __restrict__ pairs, int64_t num_pairs,
                                                                   int64_t block_vecs, int64_t src_blocks,
                                                                   int64_t dst_blocks) {
    const uint4* sbase = blockIdx.z ? src_v : src_k;
    uint4* dbase = blockIdx.z ? dst_v : dst_k;
    const int64_t first = static_cast<int64_t>(blockIdx.x) * kCopyThreads * kCopyUnroll + threadIdx.x;
    for (int64_t p = blockIdx.y; p < num_pairs; p += gridDim.y) {
        const int64_t src = pairs[2 * p];
        const int64_t dst = pairs[2 * p + 1];
        if (src < 0 || src >= src_blocks || dst < 0 || dst >= dst_blocks) {
            if (threadIdx.x == 0 && blockIdx.x == 0 && blockIdx.z == 0) flag_error(PKV_DEVERR_PAIR);
            continue;
        }
        const uint4* s = sbase + src * block_vecs;
        uint4* d = dbase + dst * block_vecs;
        uint4 r[kCopyUnroll];
#pragma unroll
        for (int u = 0; u < kCopyUnroll; ++u) {
            const int64_t i = first + u * kCopyThreads;
            if (i < block_vecs) r[u] = s[i];
        }
#pragma unroll
        for (int u = 0; u < kCopyUnroll; ++u) {
            const int64_t i = first + u * kCopyThreads;
            if (i < block_vecs) d[i] = r[u];
        }
    }
}

}  // namespace pkv
