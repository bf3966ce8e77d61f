// prefill.cuh -- causal chunked-prefill attention over the paged cache on the
// tcgen05 tensor cores.
//
// One CTA (128 threads) per (chunk, query tile, KV head).  A query tile is
// 128 rows = 128/G query tokens x the G query heads that share the KV head, so
// every K/V tile staged in shared memory serves all of them.  Per key tile of
// 128 keys (128/B physical blocks, each fetched by its own TMA box through the
// block table):
//   S  = Q . K^T        tcgen05.mma, A = Q (K-major), B = K tile (K-major),
//                        M = 128, N = 128, accumulator in tensor memory;
//   P  = exp2(S*scale*log2e - m)   one thread per row reads its row of S from
//                        tensor memory, keeps the running max / sum, writes P
//                        (input dtype) into shared memory in the 128-byte
//                        swizzled K-major layout;
//   O_t = P . V          tcgen05.mma, A = P (K-major), B = V tile (MN-major),
//                        N = head_dim, into a second tensor-memory region
//                        (bf16: P as hi + lo terms, two MMAs per K step);
//   O  = O * alpha + O_t kept in registers (one row per thread).
// K/V tiles are double-buffered: the TMA for tile j+2 is issued as soon as
// the P.V product of tile j has consumed its buffer.
#pragma once

#include "ptx.cuh"

namespace pkv {

struct PrefillParams {
    void* out;
    const int32_t* block_tables;
    const int32_t* seq_lens;
    const int32_t* query_start_loc;
    float scale_log2;
    int num_chunks;
    int num_q_heads;
    int num_kv_heads;
    int max_blocks_per_seq;
    int block_size;  // divides 128
    int64_t num_blocks;
    int q_tiles;  // query tiles per chunk in the grid
};

constexpr int kPrefillThreads = 128;

template <typename T, int D, int G>
struct PrefillCfg {
    static constexpr int BM = 128;         // rows per tile
    static constexpr int TT = BM / G;      // query tokens per tile
    static constexpr int BN = 128;         // keys per tile
    static constexpr int NP = D / 64;      // 128-byte panels per row (16-bit types)
    static constexpr int PANEL = 64;
    static constexpr int Q_BYTES = NP * BM * 128;
    static constexpr int KT_BYTES = NP * BN * 128;
    static constexpr int STAGE = 2 * KT_BYTES;
    static constexpr int P_BYTES = (BN / 64) * BM * 128;
    // bf16 keeps only 8 significant bits: P goes to the tensor cores as two
    // bf16 terms (P = hi + lo, |lo| <= 2^-8 |P|), which brings the rounding of
    // the attention weights below the output tolerance.  fp16 P is one term.
    static constexpr bool SPLIT_P = Elem<T>::kCuType == CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    static constexpr int Q_OFF = 0;
    static constexpr int ST_OFF = Q_OFF + Q_BYTES;
    static constexpr int P_OFF = ST_OFF + 2 * STAGE;
    static constexpr int PLO_OFF = P_OFF + P_BYTES;
    static constexpr int BAR_OFF = PLO_OFF + (SPLIT_P ? P_BYTES : 0);
    static constexpr int SMEM = 1024 + BAR_OFF + 64;
    static constexpr uint32_t TMEM_COLS = 256;
    static constexpr uint32_t S_COL = 0;
    static constexpr uint32_t O_COL = 128;
    static_assert(D == 64 || D == 128, "head_dim");
};

template <typename T, int D, int G>
__global__ void __launch_bounds__(kPrefillThreads, 1) paged_prefill_kernel(const PrefillParams p,
                                                                         const __grid_constant__ CUtensorMap tm_q,
                                                                         const __grid_constant__ CUtensorMap tm_k,
                                                                         const __grid_constant__ CUtensorMap tm_v) {
    using C = PrefillCfg<T, D, G>;
    const int B = p.block_size;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align_1024(smem_raw);
    uint8_t* q_s = smem + C::Q_OFF;
    uint8_t* p_s = smem + C::P_OFF;
    uint8_t* plo_s = smem + C::PLO_OFF;
    uint64_t* bar_q = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF);
    uint64_t* bar_kv = bar_q + 1;  // [2]
    uint64_t* bar_s = bar_q + 3;
    uint64_t* bar_o = bar_q + 4;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_q + 5);

    const int per_chunk = p.q_tiles * p.num_kv_heads;
    const int r = blockIdx.x / per_chunk;
    const int rem = blockIdx.x - r * per_chunk;
    const int qt = rem / p.num_kv_heads;
    const int g = rem - qt * p.num_kv_heads;
    const int tid = threadIdx.x;
    const int warp = tid >> 5;

    const int q0 = p.query_start_loc[r];
    const int n = p.query_start_loc[r + 1] - q0;
    const int L = p.seq_lens[r];
    const int c0 = L - n;
    if (n < 0 || c0 < 0 || L > p.max_blocks_per_seq * B || n > p.q_tiles * C::TT) {
        if (tid == 0 && qt == 0 && g == 0) flag_error(PKV_DEVERR_LENGTH);
        if (n < 0 || c0 < 0 || L > p.max_blocks_per_seq * B) return;
    }
    if (qt * C::TT >= n) return;
    const int tile_tokens = min(C::TT, n - qt * C::TT);
    const int kmax = c0 + qt * C::TT + tile_tokens - 1;  // last key any row of the tile needs
    const int nkt = kmax / C::BN + 1;
    const int nblk = (L + B - 1) / B;
    const int32_t* bt_row = p.block_tables + static_cast<int64_t>(r) * p.max_blocks_per_seq;

    if (warp == 0) {
        tmem_alloc(tmem_slot, C::TMEM_COLS);
        tmem_relinquish();
    }
    if (tid == 0) {
        mbar_init(bar_q, 1);
        mbar_init(&bar_kv[0], 1);
        mbar_init(&bar_kv[1], 1);
        mbar_init(bar_s, 1);
        mbar_init(bar_o, 1);
        fence_mbar_init();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    const uint32_t t_s = tmem + lane_base + C::S_COL;
    const uint32_t t_o = tmem + lane_base + C::O_COL;

    auto issue_kv = [&](int j) {  // thread 0 only
        const int st = j & 1;
        uint8_t* kd = smem + C::ST_OFF + st * C::STAGE;
        uint8_t* vd = kd + C::KT_BYTES;
        mbar_arrive_expect_tx(&bar_kv[st], C::STAGE);
#pragma unroll 1
        for (int i = 0; i < C::BN / B; ++i) {
            const int lb = j * (C::BN / B) + i;
            int id = lb < nblk ? bt_row[lb] : -1;
            if (lb < nblk && (id < 0 || id >= p.num_blocks)) {
                flag_error(PKV_DEVERR_BLOCK_ID);
                id = -1;
            }
            const int coord = id >= 0 ? id : static_cast<int>(p.num_blocks);  // out of range: zero fill
#pragma unroll
            for (int pn = 0; pn < C::NP; ++pn) {
                tma_load_4d(kd + pn * C::BN * 128 + i * B * 128, &tm_k, pn * C::PANEL, g, 0, coord, &bar_kv[st]);
                tma_load_4d(vd + pn * C::BN * 128 + i * B * 128, &tm_v, pn * C::PANEL, g, 0, coord, &bar_kv[st]);
            }
        }
    };

    if (tid == 0) {
        mbar_arrive_expect_tx(bar_q, C::Q_BYTES);
#pragma unroll
        for (int pn = 0; pn < C::NP; ++pn)
            tma_load_3d(q_s + pn * C::BM * 128, &tm_q, pn * C::PANEL, g * G, q0 + qt * C::TT, bar_q);
        issue_kv(0);
        if (nkt > 1) issue_kv(1);
    }

    // this thread's row
    const int row = tid;
    const int tok = qt * C::TT + row / G;
    const int qpos = c0 + tok;  // absolute position of the row's query
    constexpr bool kBf16 = sizeof(T) == 2 && Elem<T>::kCuType == CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    constexpr uint32_t IDESC_S = umma_idesc_f16(128, C::BN, kBf16, false, false);
    constexpr uint32_t IDESC_O = umma_idesc_f16(128, D, kBf16, false, true);
    const uint32_t q_addr = smem_u32(q_s);
    const uint32_t p_addr = smem_u32(p_s);
    const uint32_t plo_addr = smem_u32(plo_s);

    float o[D];
#pragma unroll
    for (int d = 0; d < D; ++d) o[d] = 0.f;
    float m = -INFINITY, lsum = 0.f;

    // Every wait below is bounded; its outcome is made CTA-uniform so that all
    // threads leave the loop together.  `pending` records an MMA still in
    // flight when a wait gave up (1: Q.K^T, 2: P.V).
    bool ok = !__syncthreads_or(!mbar_wait(bar_q, 0));
    int pending = 0;
    int j = 0;
    for (; ok && j < nkt; ++j) {
        const int st = j & 1;
        uint8_t* ks = smem + C::ST_OFF + st * C::STAGE;
        uint8_t* vs = ks + C::KT_BYTES;
        if (__syncthreads_or(!mbar_wait(&bar_kv[st], (j >> 1) & 1))) {
            ok = false;
            break;
        }
        // Keys at or past L inside the last live block hold no token: zero
        // their V rows so that 0-weighted garbage cannot reach the output.
        const int tile_k0 = j * C::BN;
        const int dead_lo = max(L, tile_k0), dead_hi = min(nblk * B, tile_k0 + C::BN);
        if (dead_lo < dead_hi) {
            const int rows = dead_hi - dead_lo;
            for (int i = tid; i < rows * C::NP * 8; i += kPrefillThreads) {
                const int rr = (dead_lo - tile_k0) + i / (C::NP * 8);
                const int rest = i % (C::NP * 8);
                *reinterpret_cast<uint4*>(vs + (rest / 8) * C::BN * 128 + rr * 128 + (rest % 8) * 16) =
                    make_uint4(0, 0, 0, 0);
            }
            fence_proxy_async();
        }
        tc_fence_before();
        __syncthreads();
        if (tid == 0) {
            tc_fence_after();
            const uint32_t k_addr = smem_u32(ks);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                const uint32_t off = (kk / 4) * (C::BM * 128) + (kk % 4) * 32;
                const uint32_t koff = (kk / 4) * (C::BN * 128) + (kk % 4) * 32;
                umma_f16_ss(t_s - lane_base, smem_desc_sw128(q_addr + off, 16, 1024),
                            smem_desc_sw128(k_addr + koff, 16, 1024), IDESC_S, kk > 0);
            }
            umma_commit(bar_s);
        }
        if (__syncthreads_or(!mbar_wait(bar_s, j & 1))) {
            ok = false;
            pending = 1;
            break;
        }
        tc_fence_after();

        // ---- softmax on this thread's row of S (two passes over tensor memory)
        float v[32];
        float mloc = -INFINITY;
#pragma unroll
        for (int c = 0; c < C::BN / 32; ++c) {
            tmem_ld32(t_s + c * 32, v);
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                const int key = tile_k0 + c * 32 + i;
                const float sv = key <= qpos ? v[i] * p.scale_log2 : -INFINITY;
                mloc = fmaxf(mloc, sv);
            }
        }
        const float mnew = fmaxf(m, mloc);
        const float alpha = exp2f(m - mnew);
        float tsum = 0.f;
#pragma unroll
        for (int c = 0; c < C::BN / 32; ++c) {
            tmem_ld32(t_s + c * 32, v);
            uint32_t packed[16], packed_lo[16];
#pragma unroll
            for (int i = 0; i < 32; i += 2) {
                const int key = tile_k0 + c * 32 + i;
                const float p0 = key <= qpos ? exp2f(v[i] * p.scale_log2 - mnew) : 0.f;
                const float p1 = key + 1 <= qpos ? exp2f(v[i + 1] * p.scale_log2 - mnew) : 0.f;
                tsum += p0 + p1;
                packed[i / 2] = Elem<T>::pack(p0, p1);
                if constexpr (C::SPLIT_P) {
                    const float2 hi = Elem<T>::pair(packed[i / 2]);
                    packed_lo[i / 2] = Elem<T>::pack(p0 - hi.x, p1 - hi.y);
                }
            }
            // keys c*32 .. c*32+31 -> panel c/2, 16-byte chunks 4*(c%2) .. +3
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int cc = 4 * (c % 2) + q;
                const int off = (c / 2) * (C::BM * 128) + row * 128 + ((cc ^ (row & 7)) << 4);
                *reinterpret_cast<uint4*>(p_s + off) =
                    make_uint4(packed[4 * q], packed[4 * q + 1], packed[4 * q + 2], packed[4 * q + 3]);
                if constexpr (C::SPLIT_P)
                    *reinterpret_cast<uint4*>(plo_s + off) = make_uint4(packed_lo[4 * q], packed_lo[4 * q + 1],
                                                                        packed_lo[4 * q + 2], packed_lo[4 * q + 3]);
            }
        }
        lsum = lsum * alpha + tsum;
        m = mnew;
        fence_proxy_async();
        tc_fence_before();
        __syncthreads();
        if (tid == 0) {
            tc_fence_after();
            const uint32_t v_addr = smem_u32(vs);
#pragma unroll
            for (int kk = 0; kk < C::BN / 16; ++kk) {
                const uint32_t poff = (kk / 4) * (C::BM * 128) + (kk % 4) * 32;
                const uint64_t vdesc = smem_desc_sw128(v_addr + kk * 16 * 128, C::BN * 128, 1024);
                umma_f16_ss(t_o - lane_base, smem_desc_sw128(p_addr + poff, 16, 1024), vdesc, IDESC_O, kk > 0);
                if constexpr (C::SPLIT_P)
                    umma_f16_ss(t_o - lane_base, smem_desc_sw128(plo_addr + poff, 16, 1024), vdesc, IDESC_O, 1);
            }
            umma_commit(bar_o);
        }
        if (__syncthreads_or(!mbar_wait(bar_o, j & 1))) {
            ok = false;
            pending = 2;
            break;
        }
        tc_fence_after();
        if (tid == 0 && j + 2 < nkt) issue_kv(j + 2);
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
            tmem_ld32(t_o + c * 32, v);
#pragma unroll
            for (int i = 0; i < 32; ++i) o[c * 32 + i] = fmaf(o[c * 32 + i], alpha, v[i]);
        }
    }

    if (ok) {
        if (tok < n) {
            const float inv = 1.f / lsum;
            T* dst = reinterpret_cast<T*>(p.out) +
                     (static_cast<int64_t>(q0 + tok) * p.num_q_heads + static_cast<int64_t>(g) * G + row % G) * D;
#pragma unroll
            for (int d = 0; d < D; d += 8) {
                uint4 w;
                w.x = Elem<T>::pack(o[d] * inv, o[d + 1] * inv);
                w.y = Elem<T>::pack(o[d + 2] * inv, o[d + 3] * inv);
                w.z = Elem<T>::pack(o[d + 4] * inv, o[d + 5] * inv);
                w.w = Elem<T>::pack(o[d + 6] * inv, o[d + 7] * inv);
                *reinterpret_cast<uint4*>(dst + d) = w;
            }
        }
    } else if (tid == 0) {
        // A wait gave up: wait (bounded) for whatever is still in flight
        // before tensor memory and shared memory are released.
        if (pending == 1) mbar_wait(bar_s, j & 1);
        if (pending == 2) mbar_wait(bar_o, j & 1);
        for (int jj = pending ? j + 1 : j; jj < min(nkt, j + 2); ++jj) mbar_wait(&bar_kv[jj & 1], (jj >> 1) & 1);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

}  // namespace pkv
