// prefill.cuh -- causal chunked-prefill attention over the paged cache on the
// tcgen05 tensor cores, warp-specialised, two query tiles per CTA.
//
// One CTA per (pair of query tiles, chunk, KV head).  A query tile is 128
// rows = 128/G query tokens x the G query heads that share the KV head; the
// CTA holds two consecutive tiles (a and b), so every K/V tile it stages in
// shared memory serves 256 rows.  Key tiles are 128 keys = 128/B physical
// blocks, each fetched by its own TMA box through the block table.
//
// Tensor memory (512 columns): S_a [0, 128), S_b [128, 256), O_a and O_b
// after them (head_dim columns each).  The attention weights P of a tile are
// written back over that tile's S columns (16-bit, two per column) and feed
// the P.V product straight from tensor memory, so P never touches shared
// memory.
//
// Roles (320 threads):
//  * warps 0-3 / 4-7 -- softmax of tile a / tile b, one thread per row (TMEM
//    lane = row).  For key tile j: read the row of S_j (128 columns), take its
//    max, write P_j = exp2(S_j * scale * log2 e - m) over the S columns as
//    f16, rescale O when the row max grew by more than 2^8 (lazy rescaling),
//    and signal the MMA warp.  With bf16 inputs each warpgroup then widens
//    its half of the next V tile to f16 (times 2^-8) in shared memory, so
//    that P.V runs as one f16 product.
//  * warp 8 -- loader: the two Q tiles once, then K_j (two stages) and V_j
//    (three stages for bf16, running one tile ahead of K) as soon as the MMAs
//    that read the stage's previous tile are done.  Its lanes prefetch the
//    next tile's block ids, one per lane.
//  * warp 9 -- MMA issue (lane 0), in the order
//        S_a(0) S_b(0) | PV_a(0) S_a(1) PV_b(0) S_b(1) | PV_a(1) S_a(2) ...
//    so that while one tile's softmax runs, the tensor cores work on the
//    other tile.  S_x(j+1) overwrites the columns P_x(j) occupied; it is
//    issued after PV_x(j), and tcgen05 MMAs of one thread run in order.
// Every wait is bounded; a wait that gives up raises a CTA-wide abort flag
// that ends the other roles' waits too, and every role then waits (bounded)
// for the copies / MMAs it issued before tensor memory is released.
#pragma once

#include "ptx.cuh"

namespace pkv {

struct PrefillParams {
    void* out;
    const int32_t* block_tables;
    const int32_t* seq_lens;
    const int32_t* query_start_loc;
    float scale_log2;  // scale * log2(e) (times the K pool's scale for widened FP8 pools)
    float out_scale;   // the V pool's scale for widened FP8 pools, else 1
    int num_chunks;
    int num_q_heads;
    int num_kv_heads;
    int max_blocks_per_seq;
    int block_size;  // divides 128
    int64_t num_blocks;
    int tile_pairs;  // pairs of query tiles per chunk in the grid
};

constexpr int kPrefillSoftmaxWarps = 8;                    // 4 per query tile, one thread per row
constexpr int kPrefillLoadWarp = kPrefillSoftmaxWarps;      // TMA loads of Q, K, V tiles
constexpr int kPrefillMmaWarp = kPrefillSoftmaxWarps + 1;   // tcgen05.mma issue
constexpr int kPrefillThreads = (kPrefillSoftmaxWarps + 2) * 32;

template <typename T, int D, int G>
struct PrefillCfg {
    static constexpr int BM = 128;         // rows per query tile
    static constexpr int TT = BM / G;      // query tokens per tile
    static constexpr int BN = 128;         // keys per tile
    static constexpr int NP = D / 64;      // 128-byte panels per row (16-bit types)
    static constexpr int PANEL = 64;
    static constexpr int Q_BYTES = NP * BM * 128;   // one query tile
    static constexpr int KT_BYTES = NP * BN * 128;  // one K (or V) tile
    // P.V runs in f16: P (below 2^8 under lazy rescaling) keeps 11
    // significant bits, far below the output tolerance.  bf16 V tiles are
    // widened in shared memory first, scaled by 2^-8 (exact for |v| in
    // [2^-6, 1.6e7]; below, f16 subnormals keep an absolute error under
    // 2^-25 * 2^8 = 7.6e-6; above 1.6e7 a value becomes inf); the epilogue
    // scales O back by 2^8.  Q.K^T stays in the input type.
    static constexpr bool WIDEN_V = Elem<T>::kCuType == CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    // V stages: a stage is refilled once the P.V MMAs of its tile are done;
    // widened tiles need a third stage to cover the conversion as well
    static constexpr int NV = WIDEN_V ? 3 : 2;
    static constexpr int Q_OFF = 0;                       // [2] query tiles
    static constexpr int K_OFF = Q_OFF + 2 * Q_BYTES;     // [2] stages
    static constexpr int V_OFF = K_OFF + 2 * KT_BYTES;    // [NV] stages
    static constexpr int BAR_OFF = V_OFF + NV * KT_BYTES;
    static constexpr int NBAR = 24;
    static constexpr int SMEM = 1024 + BAR_OFF + NBAR * 8;
    static constexpr uint32_t TMEM_COLS = 512;
    static constexpr uint32_t S_COL0 = 0;        // S (then P) of tile x at S_COL0 + 128 x
    static constexpr uint32_t O_COL0 = 256;      // O of tile x at O_COL0 + D x
    static_assert(D == 64 || D == 128, "head_dim");
    static_assert(SMEM <= 227 * 1024, "shared memory");
};

// 16 consecutive 32-bit columns of this thread's TMEM lane (32x32b shape);
// no wait: the caller issues tcgen05.wait::st before the data is relied on.
__device__ __forceinline__ void tmem_st16_nowait(uint32_t taddr, const uint32_t (&v)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]),
        "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
        : "memory");
}

__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// 32 consecutive 32-bit columns of this thread's TMEM lane, without the wait.
__device__ __forceinline__ void tmem_ld32_nowait(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]),
          "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]),
          "=r"(r[30]), "=r"(r[31])
        : "r"(taddr)
        : "memory");
}

// D[tmem] (+)= A[tmem] x B[smem], kind::f16: A (M x K, K packed two per
// 32-bit column, row m in lane m) read from tensor memory.
__device__ __forceinline__ void umma_f16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Work order of the CTAs: with at most kLptChunks chunks, chunks by length
// (seq_lens) descending, ties by index, and each chunk's tile pairs last pair
// first -- the longest CTAs start in the first wave and the short ones fill
// the tail (a chunk's c0 sets its CTAs' key range far more than the pair
// index does).  Every warp computes the order for itself (O(R^2 / 32) per
// lane), so no barrier is needed.  Returns false when the CTA has no item.
constexpr int kLptChunks = 64;

__device__ __forceinline__ bool prefill_item(const int32_t* seq_lens, const int32_t* qsl, int num_chunks, int tt,
                                             int max_pairs, int k, int& r_out, int& pair_out) {
    const int lane = threadIdx.x & 31;
    // a chunk's tile pairs, at most the grid's (a longer chunk is flagged and
    // cut); a chunk of negative length gets one item, which flags it
    auto pairs_of = [&](int r) {
        const int n = qsl[r + 1] - qsl[r];
        return n < 0 ? 1 : min(max_pairs, ((n + tt - 1) / tt + 1) / 2);
    };
    int found = 0, fr = 0, fpair = 0;
    for (int r = lane; r < num_chunks; r += 32) {
        const int Lr = seq_lens[r];
        int start = 0;  // tile pairs of the chunks ahead of r in the order
        for (int q = 0; q < num_chunks; ++q) {
            const int Lq = seq_lens[q];
            if (Lq > Lr || (Lq == Lr && q < r)) start += pairs_of(q);
        }
        const int pr = pairs_of(r);
        if (k >= start && k < start + pr) found = 1, fr = r, fpair = pr - 1 - (k - start);
    }
    const unsigned who = __ballot_sync(0xffffffffu, found);
    if (!who) return false;
    const int src = __ffs(who) - 1;
    r_out = __shfl_sync(0xffffffffu, fr, src);
    pair_out = __shfl_sync(0xffffffffu, fpair, src);
    return true;
}

// Two bf16 values -> two f16 values times 2^-8 (the scaling is exact; f16
// rounds the values below 2^-6 to its subnormal grid).
__device__ __forceinline__ uint32_t widen_bf16x2_scaled(uint32_t u) {
    const float lo = __uint_as_float(u << 16) * 0.00390625f;
    const float hi = __uint_as_float(u & 0xFFFF0000u) * 0.00390625f;
    return pack_half2(lo, hi);
}

__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}
__device__ __forceinline__ float fmin3(float a, float b, float c) {
    float d;
    asm("min.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

// T: the type of the query and the K/V tiles the MMAs read; TO: the output's.
template <typename T, int D, int G, typename TO = T>
__global__ void __launch_bounds__(kPrefillThreads, 1) paged_prefill_kernel(const PrefillParams p,
                                                                         const __grid_constant__ CUtensorMap tm_q,
                                                                         const __grid_constant__ CUtensorMap tm_k,
                                                                         const __grid_constant__ CUtensorMap tm_v) {
    using C = PrefillCfg<T, D, G>;
    const int B = p.block_size;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align_1024(smem_raw);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF);
    constexpr int NV = C::NV;
    uint64_t* q_full = bars + 0;
    uint64_t* k_full = bars + 1;    // [2]  TMA landed
    uint64_t* k_free = bars + 3;    // [2]  the S MMAs that read the stage are done (tcgen05.commit)
    uint64_t* v_full = bars + 5;    // [NV]
    uint64_t* v_free = bars + 8;    // [NV] the P.V MMAs that read the stage are done
    uint64_t* v_ready = bars + 11;  // [NV] the V tile widened to f16 (256 arrivals; bf16 inputs)
    uint64_t* s_full = bars + 14;   // [2]  per tile: S_x(j) done
    uint64_t* p_full = bars + 16;   // [2]  per tile: P_x(j) written (128 arrivals)
    uint64_t* o_full = bars + 18;   // [2]  per tile: the tile's last P.V done
    uint64_t* mma_done = bars + 20;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 21);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 22);

    // The CTA's (chunk, tile pair): KV head fastest; items longest first (see
    // prefill_item), or with many chunks, tile pair outermost, last pair first.
    const int g = static_cast<int>(blockIdx.x) % p.num_kv_heads;
    const int item = static_cast<int>(blockIdx.x) / p.num_kv_heads;
    int r, pair;
    if (p.num_chunks <= kLptChunks) {
        if (!prefill_item(p.seq_lens, p.query_start_loc, p.num_chunks, C::TT, p.tile_pairs, item, r, pair)) return;
    } else {
        pair = p.tile_pairs - 1 - item / p.num_chunks;
        r = item % p.num_chunks;
    }
    const int tid = threadIdx.x;
    const int warp = tid >> 5;

    const int q0 = p.query_start_loc[r];
    const int n = p.query_start_loc[r + 1] - q0;
    const int L = p.seq_lens[r];
    const int c0 = L - n;
    if (n < 0 || c0 < 0 || L > p.max_blocks_per_seq * B || n > 2 * p.tile_pairs * C::TT) {
        if (tid == 0 && pair == 0 && g == 0) flag_error(PKV_DEVERR_LENGTH);
        if (n < 0 || c0 < 0 || L > p.max_blocks_per_seq * B) return;
    }
    const int qt0 = 2 * pair;  // query tile of tile a; tile b is the next one
    if (qt0 * C::TT >= n) return;
    const bool has_b = (qt0 + 1) * C::TT < n;
    // key tiles each query tile needs: up to its last row's position
    const int nkt_a = (c0 + min((qt0 + 1) * C::TT, n) - 1) / C::BN + 1;
    const int nkt_b = has_b ? (c0 + min((qt0 + 2) * C::TT, n) - 1) / C::BN + 1 : 0;
    const int nkt = max(nkt_a, nkt_b);
    const int nblk = (L + B - 1) / B;
    const int32_t* bt_row = p.block_tables + static_cast<int64_t>(r) * p.max_blocks_per_seq;

    if (warp == 0) {
        tmem_alloc(tmem_slot, C::TMEM_COLS);
        tmem_relinquish();
    }
    if (tid == 0) {
        mbar_init(q_full, 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&k_full[i], 1);
            mbar_init(&k_free[i], 1);
            mbar_init(&s_full[i], 1);
            mbar_init(&p_full[i], 128);
            mbar_init(&o_full[i], 1);
        }
        for (int i = 0; i < NV; ++i) {
            mbar_init(&v_full[i], 1);
            mbar_init(&v_free[i], 1);
            mbar_init(&v_ready[i], 256);
        }
        mbar_init(mma_done, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    constexpr bool kBf16 = Elem<T>::kCuType == CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;

    if (warp == kPrefillLoadWarp) {
        // ================================================================ loader (whole warp, lane 0 issues)
        const int lane = tid & 31;
        const bool leader = lane == 0;
        const int per_tile = C::BN / B;  // blocks per key tile (4..16)
        // Block ids of key tile j, one per lane (lane < per_tile).  The load is
        // only issued here; its value is first used, and checked, when the tile
        // is loaded, so the table read overlaps the pipeline.
        auto fetch_ids = [&](int j) -> int {
            const int lb = j * per_tile + lane;
            return (lane < per_tile && lb < nblk) ? bt_row[lb] : -1;
        };
        auto load_tile = [&](const CUtensorMap* map, int off, uint64_t* full, int j, int ids, int nst) {
            const int st = j % nst;
            uint8_t* dst = smem + off + st * C::KT_BYTES;
            const int lb = j * per_tile + lane;
            if (lane < per_tile && lb < nblk && (ids < 0 || ids >= p.num_blocks)) {
                flag_error(PKV_DEVERR_BLOCK_ID);
                ids = -1;
            }
            if (leader) mbar_arrive_expect_tx(&full[st], C::KT_BYTES);
            for (int i = 0; i < per_tile; ++i) {
                const int id = __shfl_sync(0xffffffffu, ids, i);
                const int coord = id >= 0 ? id : static_cast<int>(p.num_blocks);  // out of range: zero fill
                if (leader) {
#pragma unroll
                    for (int pn = 0; pn < C::NP; ++pn)
                        tma_load_4d(dst + pn * C::BN * 128 + i * B * 128, map, pn * C::PANEL, g, 0, coord, &full[st]);
                }
            }
        };
        if (leader) {
            mbar_arrive_expect_tx(q_full, (has_b ? 2 : 1) * C::Q_BYTES);
            for (int x = 0; x < (has_b ? 2 : 1); ++x) {
#pragma unroll
                for (int pn = 0; pn < C::NP; ++pn)
                    tma_load_3d(smem + C::Q_OFF + x * C::Q_BYTES + pn * C::BM * 128, &tm_q, pn * C::PANEL, g * G,
                                q0 + (qt0 + x) * C::TT, q_full);
            }
        }
        int ids = fetch_ids(0);
        int j = 0;
        for (; j < min(nkt, 2); ++j) {
            load_tile(&tm_k, C::K_OFF, k_full, j, ids, 2);
            load_tile(&tm_v, C::V_OFF, v_full, j, ids, NV);
            ids = fetch_ids(j + 1);
        }
        int loaded_k = j, loaded_v = j;
        if (NV == 3 && j < nkt) {  // V runs one tile ahead of K
            load_tile(&tm_v, C::V_OFF, v_full, j, ids, NV);
            loaded_v = j + 1;
        }
        // K of tile j once the S MMAs of tile j - 2 freed its stage; V of tile
        // j + NV - 2 once the P.V MMAs of tile j - 2 did.
        for (; j < nkt; ++j) {
            const int ids_next = fetch_ids(j + 1);
            if (!__all_sync(0xffffffffu, mbar_wait_or_abort(&k_free[j & 1], ((j - 2) >> 1) & 1, abort_flag))) break;
            load_tile(&tm_k, C::K_OFF, k_full, j, ids, 2);
            loaded_k = j + 1;
            const int jv = j + NV - 2;
            if (jv < nkt) {
                if (!__all_sync(0xffffffffu, mbar_wait_or_abort(&v_free[jv % NV], ((jv - NV) / NV) & 1, abort_flag)))
                    break;
                load_tile(&tm_v, C::V_OFF, v_full, jv, NV == 2 ? ids : ids_next, NV);
                loaded_v = jv + 1;
            }
            ids = ids_next;
        }
        if (leader) {
            // Wait (bounded) for this warp's last copies: on the normal path
            // their consumers waited for them already; after an abort they may
            // still be in flight and must land before the CTA exits.
            mbar_wait(q_full, 0);
            for (int t = max(0, loaded_k - 2); t < loaded_k; ++t) mbar_wait(&k_full[t & 1], (t >> 1) & 1);
            for (int t = max(0, loaded_v - NV); t < loaded_v; ++t) mbar_wait(&v_full[t % NV], (t / NV) & 1);
        }
    } else if (warp == kPrefillMmaWarp) {
        // ================================================================ MMA issue (lane 0)
        if ((tid & 31) == 0) {
            constexpr uint32_t IDESC_S = umma_idesc_f16(128, C::BN, kBf16, false, false);
            constexpr uint32_t IDESC_O = umma_idesc_f16(128, D, false, false, true);  // f16 P and V
            // Shared-memory descriptors of every operand tile, made once: a
            // 16-element k slice is the tile's descriptor plus its byte offset / 16
            // (the start-address field), so issuing an MMA costs a few
            // instructions -- one thread issues fast enough for the tensor pipe
            // only without per-MMA descriptor arithmetic.
            uint64_t qdesc[2], kdesc[2], vdesc[NV];
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                qdesc[i] = smem_desc_sw128(smem_u32(smem + C::Q_OFF + i * C::Q_BYTES), 16, 1024);
                kdesc[i] = smem_desc_sw128(smem_u32(smem + C::K_OFF + i * C::KT_BYTES), 16, 1024);
            }
#pragma unroll
            for (int i = 0; i < NV; ++i)
                vdesc[i] = smem_desc_sw128(smem_u32(smem + C::V_OFF + i * C::KT_BYTES), C::BN * 128, 1024);
            auto issue_s = [&](int x, int t) {  // S_x(t) = Q_x . K_t^T
                const uint64_t qd = qdesc[x], kd = kdesc[t & 1];
                const uint32_t s_col = C::S_COL0 + 128 * x;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    constexpr int kQ = C::BM * 128 / 16, kK = C::BN * 128 / 16;  // panel strides / 16
                    umma_f16_ss(tmem + s_col, qd + (kk / 4) * kQ + (kk % 4) * 2, kd + (kk / 4) * kK + (kk % 4) * 2,
                                IDESC_S, kk > 0);
                }
                umma_commit(&s_full[x]);
            };
            // O_x += P_x(t) . V_t, P from tensor memory.  Only the tile's last
            // P.V is committed on its own (for the epilogue): the commit of
            // S_x(t + 1), issued after PV_x(t), also tells the softmax that O_x
            // holds every P.V before it.
            auto issue_pv = [&](int x, int t, bool last) {
                const uint64_t vd = vdesc[t % NV];
                const uint32_t p_col = C::S_COL0 + 128 * x, o_col = C::O_COL0 + D * x;
#pragma unroll
                for (int kk = 0; kk < C::BN / 16; ++kk) {
                    const uint64_t v = vd + kk * (16 * 128 / 16);  // 16 key rows of 128 bytes
                    umma_f16_ts(tmem + o_col, tmem + p_col + kk * 8, v, IDESC_O, t > 0 || kk > 0);
                }
                if (last) umma_commit(&o_full[x]);
            };
            bool ok = mbar_wait_or_abort(q_full, 0, abort_flag) && mbar_wait_or_abort(&k_full[0], 0, abort_flag);
            if (ok) {
                tc_fence_after();
                issue_s(0, 0);
                if (nkt_b > 0) issue_s(1, 0);
                umma_commit(&k_free[0]);
            }
            for (int t = 0; ok && t < nkt; ++t) {
                const bool next = t + 1 < nkt;
                bool k_next = false;  // K_{t+1} landed (waited for once, when first needed)
                ok = mbar_wait_or_abort(C::WIDEN_V ? &v_ready[t % NV] : &v_full[t % NV], (t / NV) & 1, abort_flag);
                for (int x = 0; ok && x < 2; ++x) {
                    const int nk = x == 0 ? nkt_a : nkt_b;
                    if (t >= nk) continue;
                    ok = mbar_wait_or_abort(&p_full[x], t & 1, abort_flag);
                    if (!ok) break;
                    tc_fence_after();
                    issue_pv(x, t, t + 1 == nk);
                    if (t + 1 < nk) {
                        if (!k_next) {
                            ok = k_next = mbar_wait_or_abort(&k_full[(t + 1) & 1], ((t + 1) >> 1) & 1, abort_flag);
                            if (!ok) break;
                            tc_fence_after();
                        }
                        issue_s(x, t + 1);
                    }
                }
                if (ok) {
                    umma_commit(&v_free[t % NV]);
                    if (next) umma_commit(&k_free[(t + 1) & 1]);
                }
            }
            // Wait (bounded) for every MMA this thread issued before tensor
            // memory is released: complete already on the normal path, possibly
            // in flight after an abort raised by another role.
            umma_commit(mma_done);
            mbar_wait(mma_done, 0);
        }
    } else {
        // ================================================================ softmax: one thread per row
        const int x = warp >> 2;                    // query tile of this warpgroup
        const int row = (warp & 3) * 32 + (tid & 31);
        const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
        const int tok = (qt0 + x) * C::TT + row / G;
        const int qpos = c0 + tok;  // absolute position of the row's query
        const int nk = x == 0 ? nkt_a : nkt_b;
        const uint32_t ts = tmem + lane_base + C::S_COL0 + 128 * x;
        const uint32_t to = tmem + lane_base + C::O_COL0 + D * x;
        const float sl2 = p.scale_log2;
        // Lazy rescaling: the exponent base m_used moves (and O, lsum are
        // rescaled) only when a tile's row max exceeds it by more than
        // kRescaleLog2; until then the weights exp2(s - m_used) stay below
        // 2^kRescaleLog2, far inside fp32 and the 16-bit P range.
        constexpr float kRescaleLog2 = 8.f;
        float m_used = -INFINITY, lsum = 0.f;
        bool ok = true;
        // The warpgroup whose P.V comes first for the CTA's last key tile
        // zeroes that tile's V rows past the sequence end (0 * NaN must not
        // reach O): tile a's, unless tile a stops one key tile earlier.
        const int jz = nkt - 1;
        const bool zeroes = (x == 0) == (jz < nkt_a);
        // bf16 inputs: this warpgroup's half of V tile jt's bytes (at head_dim
        // 128, one of its two panels) to f16 times 2^-8, in place; the rows past
        // the sequence end of the CTA's last key tile are zeroed instead.  Each
        // warpgroup widens V(0) first and V(j + 1) after its P(j), while the
        // tensor cores run P.V(j) and S(j + 1); P.V(j) waits for both halves.
        auto widen_half = [&](int jt) -> bool {
            if (!__all_sync(0xffffffffu, mbar_wait_or_abort(&v_full[jt % NV], (jt / NV) & 1, abort_flag)))
                return false;
            uint8_t* vs = smem + C::V_OFF + (jt % NV) * C::KT_BYTES;
            const int tk0 = jt * C::BN;
            const bool last = jt == nkt - 1;
            const int dead_lo = last ? max(L, tk0) - tk0 : C::BN;  // tile rows [dead_lo, dead_hi)
            const int dead_hi = last ? min(nblk * B, tk0 + C::BN) - tk0 : C::BN;
            constexpr int HALF = C::KT_BYTES / 2;
#pragma unroll 4
            for (int off = x * HALF + row * 16; off < (x + 1) * HALF; off += 128 * 16) {
                const int vrow = (off % (C::BN * 128)) / 128;
                uint4 v = *reinterpret_cast<const uint4*>(vs + off);
                if (vrow >= dead_lo && vrow < dead_hi) {
                    v = make_uint4(0, 0, 0, 0);
                } else {
                    v.x = widen_bf16x2_scaled(v.x);
                    v.y = widen_bf16x2_scaled(v.y);
                    v.z = widen_bf16x2_scaled(v.z);
                    v.w = widen_bf16x2_scaled(v.w);
                }
                *reinterpret_cast<uint4*>(vs + off) = v;
            }
            fence_proxy_async();  // the widened half -> the tensor cores' (async) proxy
            mbar_arrive(&v_ready[jt % NV]);
            return true;
        };
        if constexpr (C::WIDEN_V) ok = nkt > 0 && widen_half(0);
        for (int j = 0; ok && j < nk; ++j) {
            if (!__all_sync(0xffffffffu, mbar_wait_or_abort(&s_full[x], j & 1, abort_flag))) {
                ok = false;
                break;
            }
            tc_fence_after();
            float sv[C::BN];
            {
                uint32_t u[C::BN];
#pragma unroll
                for (int c = 0; c < C::BN / 32; ++c)
                    tmem_ld32_nowait(ts + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&u[c * 32]));
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < C::BN; ++i) sv[i] = __uint_as_float(u[i]);
            }
            const int k0 = j * C::BN;
            const bool all_vis = k0 + C::BN - 1 <= qpos;
            // ---- row max: raw scores on a fully visible tile (the scale goes
            // into the exponent's FMA), scaled scores with -inf masks otherwise
            float mrow;
            if (all_vis) {
                // four independent chains of 3-input max (min for a negative scale)
                float r0 = sv[0], r1 = sv[1], r2 = sv[2], r3 = sv[3];
                if (sl2 >= 0.f) {
#pragma unroll
                    for (int i = 4; i < C::BN; i += 8)
                        r0 = fmax3(r0, sv[i], sv[i + 4]), r1 = fmax3(r1, sv[i + 1], sv[i + 5]),
                        r2 = fmax3(r2, sv[i + 2], sv[i + 6]), r3 = fmax3(r3, sv[i + 3], sv[i + 7]);
                    mrow = fmaxf(fmaxf(r0, r1), fmaxf(r2, r3)) * sl2;
                } else {
#pragma unroll
                    for (int i = 4; i < C::BN; i += 8)
                        r0 = fmin3(r0, sv[i], sv[i + 4]), r1 = fmin3(r1, sv[i + 1], sv[i + 5]),
                        r2 = fmin3(r2, sv[i + 2], sv[i + 6]), r3 = fmin3(r3, sv[i + 3], sv[i + 7]);
                    mrow = fminf(fminf(r0, r1), fminf(r2, r3)) * sl2;
                }
            } else {
                float r0 = -INFINITY, r1 = -INFINITY;
#pragma unroll
                for (int i = 0; i < C::BN; i += 2) {
                    sv[i] = k0 + i <= qpos ? sv[i] * sl2 : -INFINITY;
                    sv[i + 1] = k0 + i + 1 <= qpos ? sv[i + 1] * sl2 : -INFINITY;
                    r0 = fmaxf(r0, sv[i]);
                    r1 = fmaxf(r1, sv[i + 1]);
                }
                mrow = fmaxf(r0, r1);
            }
            const bool rescale = mrow > m_used + kRescaleLog2 || (m_used == -INFINITY && mrow != -INFINITY);
            float alpha = 1.f;
            if (rescale) {
                alpha = ex2_approx(m_used - mrow);  // 0 when m_used is -inf
                m_used = mrow;
            }
            const float mexp = m_used == -INFINITY ? 0.f : m_used;
            const float smul = all_vis ? sl2 : 1.f;  // the exponent is sv * smul - m
            // ---- P = exp2(S - m_used) over the S columns, 32 keys at a time
            // (packed f32x2 arithmetic: the exponent arguments and the row sum)
            float2 acc[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
            const float2 smul2 = make_float2(smul, smul), nm2 = make_float2(-mexp, -mexp);
#pragma unroll
            for (int c = 0; c < C::BN / 32; ++c) {
                uint32_t pw[16];  // f16 pairs
#pragma unroll
                for (int i = 0; i < 32; i += 2) {
                    const float2 arg = __ffma2_rn(make_float2(sv[c * 32 + i], sv[c * 32 + i + 1]), smul2, nm2);
                    const float p0 = ex2_approx(arg.x), p1 = ex2_approx(arg.y);
                    acc[(i / 2) & 1] = __fadd2_rn(acc[(i / 2) & 1], make_float2(p0, p1));
                    pw[i / 2] = pack_half2(p0, p1);
                }
                tmem_st16_nowait(ts + c * 16, pw);
            }
            lsum = lsum * alpha + ((acc[0].x + acc[0].y) + (acc[1].x + acc[1].y));
            // ---- O *= alpha: P.V of the previous tile is done (S_j, committed
            // after it, was), and the next P.V accumulates on top of it
            if (j >= 1 && __any_sync(0xffffffffu, rescale && alpha != 1.f)) {
#pragma unroll
                for (int c = 0; c < D / 32; ++c) {  // warp-collective: lanes without a rescale store O back as is
                    float v[32];
                    tmem_ld32(to + c * 32, v);
#pragma unroll
                    for (int i = 0; i < 32; ++i) v[i] *= alpha;
                    tmem_st32(to + c * 32, v);
                }
            }
            // ---- dead V rows of the last key tile
            if (!C::WIDEN_V && j == jz && zeroes) {
                const int tk0 = j * C::BN;
                const int dead_lo = max(L, tk0), dead_hi = min(nblk * B, tk0 + C::BN);
                if (dead_lo < dead_hi) {
                    if (!__all_sync(0xffffffffu, mbar_wait_or_abort(&v_full[j % NV], (j / NV) & 1, abort_flag))) {
                        ok = false;
                        break;
                    }
                    uint8_t* vs = smem + C::V_OFF + (j % NV) * C::KT_BYTES;
                    const int rows = dead_hi - dead_lo;
                    for (int i = row; i < rows * C::NP * 8; i += 128) {
                        const int rr = (dead_lo - tk0) + i / (C::NP * 8);
                        const int rest = i % (C::NP * 8);
                        *reinterpret_cast<uint4*>(vs + (rest / 8) * C::BN * 128 + rr * 128 + (rest % 8) * 16) =
                            make_uint4(0, 0, 0, 0);
                    }
                    fence_proxy_async();
                }
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&p_full[x]);
            if constexpr (C::WIDEN_V) {
                if (j + 1 < nkt && !widen_half(j + 1)) {
                    ok = false;
                    break;
                }
            }
        }
        if constexpr (C::WIDEN_V) {  // tiles past this warpgroup's last (its query tile needs fewer)
            for (int jt = max(nk + 1, 1); ok && jt < nkt; ++jt) ok = widen_half(jt);
        }
        if (ok && nk > 0) {
            if (__all_sync(0xffffffffu, mbar_wait_or_abort(&o_full[x], 0, abort_flag))) {
                tc_fence_after();
                const bool live = tok < n && !*abort_flag;
                const float inv = p.out_scale * (C::WIDEN_V ? 256.f : 1.f) / lsum;
                TO* dst = reinterpret_cast<TO*>(p.out) +
                          (static_cast<int64_t>(q0 + tok) * p.num_q_heads + static_cast<int64_t>(g) * G + row % G) * D;
#pragma unroll
                for (int c = 0; c < D / 32; ++c) {
                    float v[32];
                    tmem_ld32(to + c * 32, v);  // warp-collective: every lane loads
                    if (live) {
#pragma unroll
                        for (int d = 0; d < 32; d += 8) {
                            uint4 w;
                            w.x = Elem<TO>::pack(v[d] * inv, v[d + 1] * inv);
                            w.y = Elem<TO>::pack(v[d + 2] * inv, v[d + 3] * inv);
                            w.z = Elem<TO>::pack(v[d + 4] * inv, v[d + 5] * inv);
                            w.w = Elem<TO>::pack(v[d + 6] * inv, v[d + 7] * inv);
                            *reinterpret_cast<uint4*>(dst + c * 32 + d) = w;
                        }
                    }
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

}  // namespace pkv
