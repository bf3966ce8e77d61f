// prefill.cuh -- causal chunked-prefill attention over the paged cache on the
// tcgen05 tensor cores, warp-specialised.
//
// One CTA per (query tile, chunk, KV head).  A query tile is 128 rows = 128/G
// query tokens x the G query heads that share the KV head, so every K/V tile
// staged in shared memory serves all of them.  Key tiles are 128 keys =
// 128/B physical blocks, each fetched by its own TMA box through the block
// table.
//
// Roles (288 threads):
//  * warp 8 -- producer.  A loop that polls the pipeline's mbarriers
//    (test_wait, which never suspends) issues, from lane 0,, whenever its inputs are ready and its target buffer is
//    free: the TMA loads of K and V tiles (two stages each; K of tile j+2
//    as soon as Q.K^T of tile j is done, V of tile j+2 as soon as P.V of tile
//    j is done), S_j = Q . K_j^T (tcgen05.mma, M = N = 128, into one of two
//    S buffers in tensor memory), and O_j = P_j . V_j (N = head_dim, into one
//    of two O buffers; bf16 P goes in as hi + lo terms).  The warp's lanes
//    prefetch the next tiles' block ids (one per lane) so that table reads
//    overlap the pipeline.
//  * warps 0-7 -- two threads per query row (warps w and w + 4 share TMEM lane
//    quadrant w, each takes half of the 128 key columns and half of the
//    head_dim output columns; the row max is exchanged through shared memory
//    under a pair of mbarriers per quadrant).  For tile j: read S_j from tensor
//    memory (row max), fold the finished P.V product of tile j-1 into the
//    register accumulator (online-softmax rescale), write P_j = exp2(S_j *
//    scale * log2 e - m) to shared memory in the 128-byte-swizzled K-major
//    layout, and release the S buffer.  The Q.K^T product of tile j+1 runs
//    on the tensor cores meanwhile, and P.V of tile j-1 during the max pass.
// Every wait is bounded; a wait that gives up raises a CTA-wide abort flag
// that ends the other roles' waits too.  In the softmax warps every wait
// outcome is agreed by the whole warp (the tcgen05.ld that follow are
// warp-collective).
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
    int q_tiles;  // query tiles per chunk in the grid
};

constexpr int kPrefillSoftmaxWarps = 8;  // two per TMEM lane quadrant: each row split in two column halves
constexpr int kPrefillLoadWarp = kPrefillSoftmaxWarps;      // TMA loads of K / V tiles
constexpr int kPrefillMmaWarp = kPrefillSoftmaxWarps + 1;   // tcgen05.mma issue
constexpr int kPrefillThreads = (kPrefillSoftmaxWarps + 2) * 32;

template <typename T, int D, int G>
struct PrefillCfg {
    static constexpr int BM = 128;         // rows per tile
    static constexpr int TT = BM / G;      // query tokens per tile
    static constexpr int BN = 128;         // keys per tile
    static constexpr int NP = D / 64;      // 128-byte panels per row (16-bit types)
    static constexpr int PANEL = 64;
    static constexpr int Q_BYTES = NP * BM * 128;
    static constexpr int KT_BYTES = NP * BN * 128;  // one K (or V) tile
    static constexpr int P_BYTES = (BN / 64) * BM * 128;
    // bf16 keeps only 8 significant bits: P goes to the tensor cores as two
    // bf16 terms (P = hi + lo: hi the top 16 bits of P, lo the remainder
    // rounded, |lo| < 2^-7 |P|), which brings the rounding of the attention
    // weights far below the output tolerance.  fp16 P is one term.
    static constexpr bool SPLIT_P = Elem<T>::kCuType == CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    static constexpr int Q_OFF = 0;
    static constexpr int K_OFF = Q_OFF + Q_BYTES;
    static constexpr int V_OFF = K_OFF + 2 * KT_BYTES;
    static constexpr int P_OFF = V_OFF + 2 * KT_BYTES;
    static constexpr int PLO_OFF = P_OFF + P_BYTES;
    static constexpr int BAR_OFF = PLO_OFF + (SPLIT_P ? P_BYTES : 0);
    static constexpr int NBAR = 24;
    static constexpr int XCH_OFF = BAR_OFF + NBAR * 8;      // [128 rows][2 halves] floats
    static constexpr int SMEM = 1024 + XCH_OFF + BM * 2 * 4;
    static constexpr uint32_t TMEM_COLS = 512;
    static constexpr uint32_t S_COL0 = 0, O_COL0 = 256;  // S buffers at 0 / 128, the O accumulator at 256
    static_assert(D == 64 || D == 128, "head_dim");
};

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
    uint64_t* q_full = bars + 0;
    uint64_t* k_full = bars + 1;   // [2]
    uint64_t* v_full = bars + 3;   // [2]
    uint64_t* s_full = bars + 5;   // [2]  Q.K^T done (tcgen05.commit)
    uint64_t* s_free = bars + 7;   // [2]  softmax finished reading S
    uint64_t* p_full = bars + 9;   //      P of the current tile written
    uint64_t* o_full = bars + 10;  // [2]  P.V of tile t done (tcgen05.commit), barrier t & 1
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 14);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 15);
    uint64_t* xch_full = bars + 16;  // [4]  both halves of a quadrant's rows posted a value
    uint64_t* xch_read = bars + 20;  // [4]  both halves read their partner's value

    // Launch order: query tile outermost, last tile first -- later tiles of a
    // chunk attend to more keys, so the longest CTAs start in the first wave
    // and the short ones fill the tail.
    const int ctas_per_qtile = p.num_chunks * p.num_kv_heads;
    const int qt = p.q_tiles - 1 - static_cast<int>(blockIdx.x) / ctas_per_qtile;
    const int rem = static_cast<int>(blockIdx.x) % ctas_per_qtile;
    const int r = rem / p.num_kv_heads;
    const int g = rem % p.num_kv_heads;
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
        mbar_init(q_full, 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&k_full[i], 1);
            mbar_init(&v_full[i], 1);
            mbar_init(&s_full[i], 1);
            mbar_init(&s_free[i], kPrefillSoftmaxWarps * 32);
            mbar_init(&o_full[i], 1);
        }
        mbar_init(p_full, kPrefillSoftmaxWarps * 32);
        for (int i = 0; i < 4; ++i) {
            mbar_init(&xch_full[i], 64);
            mbar_init(&xch_read[i], 64);
        }
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
        auto load_tile = [&](const CUtensorMap* map, int off, uint64_t* full, int j, int ids) {
            const int st = j & 1;
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
            mbar_arrive_expect_tx(q_full, C::Q_BYTES);
#pragma unroll
            for (int pn = 0; pn < C::NP; ++pn)
                tma_load_3d(smem + C::Q_OFF + pn * C::BM * 128, &tm_q, pn * C::PANEL, g * G, q0 + qt * C::TT, q_full);
        }
        int ids = fetch_ids(0);
        int j = 0;
        for (; j < min(nkt, 2); ++j) {
            load_tile(&tm_k, C::K_OFF, k_full, j, ids);
            load_tile(&tm_v, C::V_OFF, v_full, j, ids);
            ids = fetch_ids(j + 1);
        }
        // K of tile j once Q.K^T of tile j - 2 freed its stage; V of tile j once P.V of tile j - 2 did.
        int loaded_k = j, loaded_v = j;
        for (; j < nkt; ++j) {
            const int ids_next = fetch_ids(j + 1);
            if (!__all_sync(0xffffffffu, mbar_wait_or_abort(&s_full[j & 1], ((j - 2) >> 1) & 1, abort_flag))) break;
            load_tile(&tm_k, C::K_OFF, k_full, j, ids);
            loaded_k = j + 1;
            if (!__all_sync(0xffffffffu, mbar_wait_or_abort(&o_full[j & 1], ((j - 2) >> 1) & 1, abort_flag))) break;
            load_tile(&tm_v, C::V_OFF, v_full, j, ids);
            loaded_v = j + 1;
            ids = ids_next;
        }
        if (leader) {
            // Wait (bounded) for this warp's last copies.  On the normal path
            // their consumers already waited for them; after an abort (another
            // role's wait gave up, perhaps after this loop ended) they may
            // still be in flight and must land before the CTA exits.
            mbar_wait(q_full, 0);
            for (int t = max(0, loaded_k - 2); t < loaded_k; ++t) mbar_wait(&k_full[t & 1], (t >> 1) & 1);
            for (int t = max(0, loaded_v - 2); t < loaded_v; ++t) mbar_wait(&v_full[t & 1], (t >> 1) & 1);
        }
    } else if (warp == kPrefillMmaWarp) {
        // ================================================================ MMA issue (lane 0)
        // Order: S_0, S_1, O_0, S_2, O_1, ... -- the next tile's Q.K^T is always
        // queued ahead of the current tile's P.V.
        if ((tid & 31) == 0) {
            constexpr uint32_t IDESC_S = umma_idesc_f16(128, C::BN, kBf16, false, false);
            constexpr uint32_t IDESC_O = umma_idesc_f16(128, D, kBf16, false, true);
            const uint32_t q_addr = smem_u32(smem + C::Q_OFF);
            const uint32_t p_addr = smem_u32(smem + C::P_OFF);
            const uint32_t plo_addr = smem_u32(smem + C::PLO_OFF);
            int ns = 0, npv = 0;
            auto issue_s = [&](int t) -> bool {
                const int st = t & 1;
                if (!mbar_wait_or_abort(&k_full[st], (t >> 1) & 1, abort_flag)) return false;
                if (t >= 2 && !mbar_wait_or_abort(&s_free[st], ((t - 2) >> 1) & 1, abort_flag)) return false;
                tc_fence_after();
                const uint32_t k_addr = smem_u32(smem + C::K_OFF + st * C::KT_BYTES);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t qoff = (kk / 4) * (C::BM * 128) + (kk % 4) * 32;
                    const uint32_t koff = (kk / 4) * (C::BN * 128) + (kk % 4) * 32;
                    umma_f16_ss(tmem + C::S_COL0 + st * 128, smem_desc_sw128(q_addr + qoff, 16, 1024),
                                smem_desc_sw128(k_addr + koff, 16, 1024), IDESC_S, kk > 0);
                }
                umma_commit(&s_full[st]);
                ns = t + 1;
                return true;
            };
            // O accumulates over all key tiles in one TMEM buffer; the softmax
            // rescales it (rarely) before it posts P of the next tile.
            auto issue_pv = [&](int t) -> bool {
                const int st = t & 1;
                if (!mbar_wait_or_abort(p_full, t & 1, abort_flag)) return false;
                if (!mbar_wait_or_abort(&v_full[st], (t >> 1) & 1, abort_flag)) return false;
                tc_fence_after();
                const uint32_t v_addr = smem_u32(smem + C::V_OFF + st * C::KT_BYTES);
#pragma unroll
                for (int kk = 0; kk < C::BN / 16; ++kk) {
                    const uint32_t poff = (kk / 4) * (C::BM * 128) + (kk % 4) * 32;
                    const uint64_t vdesc = smem_desc_sw128(v_addr + kk * 16 * 128, C::BN * 128, 1024);
                    umma_f16_ss(tmem + C::O_COL0, smem_desc_sw128(p_addr + poff, 16, 1024), vdesc, IDESC_O,
                                t > 0 || kk > 0);
                    if constexpr (C::SPLIT_P)
                        umma_f16_ss(tmem + C::O_COL0, smem_desc_sw128(plo_addr + poff, 16, 1024), vdesc, IDESC_O, 1);
                }
                umma_commit(&o_full[st]);
                npv = t + 1;
                return true;
            };
            bool ok = mbar_wait_or_abort(q_full, 0, abort_flag) && issue_s(0);
            for (int t = 0; ok && t < nkt; ++t) {
                if (t + 1 < nkt) ok = issue_s(t + 1);
                if (ok) ok = issue_pv(t);
            }
            // Wait (bounded) for the MMAs this thread issued before tensor memory
            // is released: complete already on the normal path, possibly in
            // flight after an abort raised by another role.
            if (ns > 0) mbar_wait(&s_full[(ns - 1) & 1], ((ns - 1) >> 1) & 1);
            if (npv > 0) mbar_wait(&o_full[(npv - 1) & 1], ((npv - 1) >> 1) & 1);
        }
    } else {
        // ================================================================ softmax rows
        const int quad = warp & 3, half = warp >> 2;
        const int row = quad * 32 + (tid & 31);
        const int tok = qt * C::TT + row / G;
        const int qpos = c0 + tok;  // absolute position of the row's query
        const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
        constexpr int HC = C::BN / 2;  // key columns of this thread
        constexpr int HD = D / 2;      // output columns of this thread
        uint8_t* p_s = smem + C::P_OFF;
        uint8_t* plo_s = smem + C::PLO_OFF;
        float* xch = reinterpret_cast<float*>(smem + C::XCH_OFF);
        const float sl2 = p.scale_log2;
        // Lazy rescaling: the exponent base m_used moves (and O, lsum are
        // rescaled) only when a tile's row max exceeds it by more than
        // kRescaleLog2; until then the weights exp2(s - m_used) stay below
        // 2^kRescaleLog2, far inside fp32 and the 16-bit P range.
        constexpr float kRescaleLog2 = 8.f;
        float m_used = -INFINITY, lsum = 0.f;
        bool ok = true;
        float sv[HC];  // this thread's half row of S for the current tile
        float v[32];
        // Post this half's value for the row, return the partner half's (exchange
        // number e; the slot is reused once the partner read the previous one).
        auto exchange = [&](float mine, int e, float& theirs) -> bool {
            if (e > 0 &&
                !__all_sync(0xffffffffu, mbar_wait_or_abort(&xch_read[quad], (e - 1) & 1, abort_flag)))
                return false;
            xch[row * 2 + half] = mine;
            mbar_arrive(&xch_full[quad]);
            if (!__all_sync(0xffffffffu, mbar_wait_or_abort(&xch_full[quad], e & 1, abort_flag))) return false;
            theirs = xch[row * 2 + (half ^ 1)];
            mbar_arrive(&xch_read[quad]);
            return true;
        };
        const uint32_t to = tmem + lane_base + C::O_COL0 + half * HD;  // this half row of O
        for (int j = 0; j < nkt; ++j) {
            const int st = j & 1;
            if (!__all_sync(0xffffffffu, mbar_wait_or_abort(&s_full[st], (j >> 1) & 1, abort_flag))) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t ts = tmem + lane_base + C::S_COL0 + st * 128 + half * HC;
            const int k0 = j * C::BN + half * HC;  // first key of this thread's columns
            const bool all_vis = k0 + HC - 1 <= qpos;
            const bool none_vis = k0 > qpos;
            // ---- S into registers (scaled to the log2 domain, hidden keys at -inf), half-row max
            // (tcgen05.ld is warp-collective: every lane loads, masking is per row in registers)
            // A fully visible half row keeps the raw scores (the scale goes into the
            // exponent's FMA); a diagonal one holds scaled scores with -inf masks.
            float mhalf = -INFINITY;
#pragma unroll
            for (int c = 0; c < HC / 32; ++c) tmem_ld32(ts + c * 32, *reinterpret_cast<float(*)[32]>(&sv[c * 32]));
            if (all_vis) {
                // four independent chains (max and min are exact in any order)
                float r0 = sv[0], r1 = sv[1], r2 = sv[2], r3 = sv[3];
                if (sl2 >= 0.f) {
#pragma unroll
                    for (int i = 4; i < HC; i += 4)
                        r0 = fmaxf(r0, sv[i]), r1 = fmaxf(r1, sv[i + 1]), r2 = fmaxf(r2, sv[i + 2]),
                        r3 = fmaxf(r3, sv[i + 3]);
                    mhalf = fmaxf(fmaxf(r0, r1), fmaxf(r2, r3)) * sl2;
                } else {
#pragma unroll
                    for (int i = 4; i < HC; i += 4)
                        r0 = fminf(r0, sv[i]), r1 = fminf(r1, sv[i + 1]), r2 = fminf(r2, sv[i + 2]),
                        r3 = fminf(r3, sv[i + 3]);
                    mhalf = fminf(fminf(r0, r1), fminf(r2, r3)) * sl2;
                }
            } else {
#pragma unroll
                for (int i = 0; i < HC; ++i) {
                    sv[i] = k0 + i <= qpos ? sv[i] * sl2 : -INFINITY;
                    mhalf = fmaxf(mhalf, sv[i]);
                }
            }
            const float smul = all_vis ? sl2 : 1.f;  // the exponent is sv * smul - m
            tc_fence_before();
            mbar_arrive(&s_free[st]);  // S_j is in registers: its buffer may take S_{j+2}
            if (none_vis) mhalf = -INFINITY;
            float mother = -INFINITY;
            if (!exchange(mhalf, j, mother)) {
                ok = false;
                break;
            }
            const float mrow = fmaxf(mhalf, mother);
            // both halves of a row see the same (m_used, mrow) and take the same decision
            const bool rescale = mrow > m_used + kRescaleLog2 || (m_used == -INFINITY && mrow != -INFINITY);
            float alpha = 1.f;
            if (rescale) {
                alpha = ex2_approx(m_used - mrow);  // 0 when m_used is -inf
                m_used = mrow;
            }
            const float mexp = m_used == -INFINITY ? 0.f : m_used;
            // ---- P = exp2(S - m_used) for this half (= P panel `half`), into registers
            float ts4[4] = {0.f, 0.f, 0.f, 0.f};  // partial sums: four independent chains
            uint32_t hi[HC / 2], lo[C::SPLIT_P ? HC / 2 : 1];
#pragma unroll
            for (int i = 0; i < HC; i += 2) {
                const float p0 = ex2_approx(fmaf(sv[i], smul, -mexp));
                const float p1 = ex2_approx(fmaf(sv[i + 1], smul, -mexp));
                ts4[(i / 2) & 3] += p0 + p1;
                const int w = i / 2;
                if constexpr (C::SPLIT_P) {
                    // hi = p truncated to bf16 (its top 16 bits, one byte permute for the
                    // pair); lo = the exact remainder rounded to bf16, |lo| < 2^-7 |p|
                    const uint32_t b0 = __float_as_uint(p0), b1 = __float_as_uint(p1);
                    hi[w] = __byte_perm(b0, b1, 0x7632);
                    lo[w] = Elem<T>::pack(p0 - __uint_as_float(b0 & 0xFFFF0000u),
                                          p1 - __uint_as_float(b1 & 0xFFFF0000u));
                } else {
                    hi[w] = Elem<T>::pack(p0, p1);
                }
            }
            const float tsum = (ts4[0] + ts4[1]) + (ts4[2] + ts4[3]);
            lsum = lsum * alpha + tsum;  // this half's share of the row sum
            // ---- P.V of the previous tile must be done before P is overwritten (and O rescaled)
            if (j >= 1 &&
                !__all_sync(0xffffffffu, mbar_wait_or_abort(&o_full[(j - 1) & 1], ((j - 1) >> 1) & 1, abort_flag))) {
                ok = false;
                break;
            }
            if (j >= 1 && __any_sync(0xffffffffu, rescale && alpha != 1.f)) {
                tc_fence_after();
#pragma unroll
                for (int c = 0; c < HD / 32; ++c) {  // warp-collective: lanes without a rescale store O back as is
                    tmem_ld32(to + c * 32, v);
#pragma unroll
                    for (int i = 0; i < 32; ++i) v[i] *= alpha;
                    tmem_st32(to + c * 32, v);
                }
            }
            // ---- the last tile may hold the dead tail of the sequence's last
            // block: zero those V rows (0 * NaN must not reach the output)
            if (j == nkt - 1) {
                const int tk0 = j * C::BN;
                const int dead_lo = max(L, tk0), dead_hi = min(nblk * B, tk0 + C::BN);
                if (dead_lo < dead_hi) {
                    if (!__all_sync(0xffffffffu, mbar_wait_or_abort(&v_full[st], (j >> 1) & 1, abort_flag))) {
                        ok = false;
                        break;
                    }
                    uint8_t* vs = smem + C::V_OFF + st * C::KT_BYTES;
                    const int rows = dead_hi - dead_lo;
                    for (int i = tid; i < rows * C::NP * 8; i += kPrefillSoftmaxWarps * 32) {
                        const int rr = (dead_lo - tk0) + i / (C::NP * 8);
                        const int rest = i % (C::NP * 8);
                        *reinterpret_cast<uint4*>(vs + (rest / 8) * C::BN * 128 + rr * 128 + (rest % 8) * 16) =
                            make_uint4(0, 0, 0, 0);
                    }
                }
            }
#pragma unroll
            for (int q = 0; q < HC / 8; ++q) {  // 16-byte chunks of this half row
                const int off = half * (C::BM * 128) + row * 128 + ((q ^ (row & 7)) << 4);
                *reinterpret_cast<uint4*>(p_s + off) = make_uint4(hi[4 * q], hi[4 * q + 1], hi[4 * q + 2], hi[4 * q + 3]);
                if constexpr (C::SPLIT_P)
                    *reinterpret_cast<uint4*>(plo_s + off) =
                        make_uint4(lo[4 * q], lo[4 * q + 1], lo[4 * q + 2], lo[4 * q + 3]);
            }
            fence_proxy_async();
            tc_fence_before();
            mbar_arrive(p_full);
        }
        float o[HD];
        if (ok) {
            const int jl = nkt - 1;
            if (__all_sync(0xffffffffu, mbar_wait_or_abort(&o_full[jl & 1], (jl >> 1) & 1, abort_flag))) {
                tc_fence_after();
#pragma unroll
                for (int c = 0; c < HD / 32; ++c) {
                    tmem_ld32(to + c * 32, v);
#pragma unroll
                    for (int i = 0; i < 32; ++i) o[c * 32 + i] = v[i];
                }
            } else {
                ok = false;
            }
        }
        float lother = 0.f;
        if (ok && !exchange(lsum, nkt, lother)) ok = false;
        if (ok && !*abort_flag && tok < n) {
            const float inv = p.out_scale / (lsum + lother);
            TO* dst = reinterpret_cast<TO*>(p.out) +
                     (static_cast<int64_t>(q0 + tok) * p.num_q_heads + static_cast<int64_t>(g) * G + row % G) * D +
                     half * HD;
#pragma unroll
            for (int d = 0; d < HD; d += 8) {
                uint4 w;
                w.x = Elem<TO>::pack(o[d] * inv, o[d + 1] * inv);
                w.y = Elem<TO>::pack(o[d + 2] * inv, o[d + 3] * inv);
                w.z = Elem<TO>::pack(o[d + 4] * inv, o[d + 5] * inv);
                w.w = Elem<TO>::pack(o[d + 6] * inv, o[d + 7] * inv);
                *reinterpret_cast<uint4*>(dst + d) = w;
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
