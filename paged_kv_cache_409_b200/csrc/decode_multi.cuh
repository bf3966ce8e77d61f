// decode_multi.cuh -- multi-token decode: each sequence (a "chunk") holds n
// new tokens at the end of its context (speculative verification of n draft
// tokens, guide page "Speculative Decoding": a small draft model proposes the
// next tokens and the large model checks them all in one pass).  Row i of a
// chunk with c0 = seq_len - n prior tokens attends causally to keys
// j <= c0 + i -- the chunked-prefill definition, for chunks of a few tokens.
//
// A KV head serves R = n * G query rows (token-major: row r = i * G + hh),
// at most 32.  That is far below the 128-row M of a tcgen05 MMA, so the keys
// go on M and the rows on N, on the 5th-generation tensor cores:
//   S^T [128 keys x 32 rows] = K [128 keys x D] . Q^T        (A: the K tile,
//                                                             B: the Q rows)
//   O^T [D x 32 rows]       += V^T [D x 128 keys] . P^T      (A: the V tile read
//                                                             MN-major, B: P^T)
// S^T and O^T live in tensor memory (lane = key, resp. lane = head_dim
// element; column = query row).  The tensor cores then do 4 flops per K/V
// element per row in 24 (bf16: 40) instructions per 128-key tile, and the
// kernel is bound by streaming K/V from HBM.
//
// Persistent grid: one CTA per SM takes work items (chunk, partition, KV
// head) by rank blockIdx.x, blockIdx.x + gridDim.x, ...; its loader streams
// the K/V tiles of consecutive items through one ring, so an item's epilogue
// overlaps the next item's loads.  With at most kMultiLptChunks chunks the
// ranks go longest first (every full partition, then the chunks' shorter
// last partitions by key tiles, descending); else partition-major.
//
// Roles, by warp (kMultiRowGroups = 2: 16 warps, 512 threads):
//  * softmax warps (4 per row group) -- TMEM lane t (key t of a tile for
//    S^T) belongs to warp t / 32 of each row group; a row group takes
//    32 / kMultiRowGroups of the 32 rows.  For key tile j: read the key's
//    scores, mask them (causal limit, context end), and vote: when any score
//    exceeds its row's exponent base by more than 2^8 (lazy rescaling; always
//    on an item's first tile), the tile's row maxima are reduced across the
//    128 keys (warp shuffles + shared memory), the bases move and O^T is
//    rescaled in tensor memory.  Then P = exp2(s - m) goes to shared memory
//    as P^T (bf16: hi + lo terms), and per-thread partial row sums accumulate.
//    After the item's last tile the row sums are reduced the same way and
//    handed, with the rows' exponent bases, to the epilogue warps.
//  * K loader -- per item the Q rows (one TMA box per 64 dims), then the K
//    tiles (one box per physical block and 64 dims) into two stages;
//    V loader (the last warp) -- the V tiles into three.
//  * S issuer, P.V issuer (lane 0 each) -- the S^T MMAs of each tile as soon
//    as its K stage and S buffer are ready; the P.V MMAs as soon as P^T and
//    the V stage are.  The softmax of tile j runs while S(j+1) and PV(j-1) run.
//  * 4 epilogue warps, thread t = O^T lane t -- after the item's last P.V,
//    element t of every row (or of the partition's partial, for the merge
//    kernel), while the softmax goes on with the next item.
// Every wait is bounded; a wait that gives up raises a CTA-wide abort flag,
// the softmax warps leave their loop together (their named barriers stay
// matched), and every role waits (bounded) for the copies / MMAs it issued
// before tensor memory is released.
#pragma once

#include "decode.cuh"

namespace pkv {

struct MultiParams {
    void* out;                       // [total_q_tokens, Hq, D]
    const int32_t* block_tables;     // [num_chunks, max_blocks_per_seq]
    const int32_t* seq_lens;         // [num_chunks]
    const int32_t* query_start_loc;  // [num_chunks + 1]
    float* ws_max;                   // [total_q_tokens, Hq, P] (log2 domain)
    float* ws_sum;                   // [total_q_tokens, Hq, P]
    float* ws_out;                   // [total_q_tokens, Hq, P, D]
    float scale_log2;
    int num_chunks;
    int num_q_heads;
    int num_kv_heads;
    int group;  // G = num_q_heads / num_kv_heads; n * G <= 32 rows per chunk
    int block_size;
    int max_blocks_per_seq;
    int64_t num_blocks;
    int partition_blocks;
    int num_partitions;
    int64_t total_q_tokens;
};

// Softmax warps per TMEM lane quadrant, each with 32 / kMultiRowGroups of the 32 rows.
#ifndef PKV_MULTI_ROW_GROUPS
#define PKV_MULTI_ROW_GROUPS 4
#endif
constexpr int kMultiRowGroups = PKV_MULTI_ROW_GROUPS;
constexpr int kMultiRPT = 32 / kMultiRowGroups;  // rows per softmax thread
constexpr int kMultiSoftmaxWarps = 4 * kMultiRowGroups;
constexpr int kMultiSoftmaxThreads = kMultiSoftmaxWarps * 32;
static_assert(kMultiRowGroups == 2 || kMultiRowGroups == 4, "row groups");
constexpr int kMultiLoadWarp = kMultiSoftmaxWarps;
constexpr int kMultiMmaSWarp = kMultiSoftmaxWarps + 1;   // issues the S^T MMAs
constexpr int kMultiMmaPVWarp = kMultiSoftmaxWarps + 2;  // issues the P.V MMAs
constexpr int kMultiEpiWarp0 = kMultiSoftmaxWarps + 3;   // 4 epilogue warps (one per TMEM lane quadrant)
constexpr int kMultiLoadVWarp = kMultiSoftmaxWarps + 7;  // loads the V tiles (kMultiLoadWarp: the Q rows and K tiles)
constexpr int kMultiThreads = (kMultiSoftmaxWarps + 8) * 32;
constexpr int kMultiLptChunks = 128;  // up to this many chunks the items go longest first
constexpr int kMultiKT = 128;         // keys per tile
constexpr int kMultiItemCache = 32;   // items a CTA decodes once, at its start

template <int D>
struct MultiCfg {
    static constexpr int KT = kMultiKT;        // keys per tile (M of S^T)
    static constexpr int NR = 32;              // query rows per KV head (N of both products)
    static constexpr int NP = D / 64;          // 128-byte panels of a 16-bit row
    static constexpr int TILE = NP * KT * 128;  // one K (or V) tile
    // Stages of K (refilled once S(t) is done; the S MMAs run well ahead of
    // the softmax) and of V (refilled once PV(t) is done, which waits for the
    // softmax of tile t: three stages cover the load latency).
    static constexpr int NSK = 2;
    static constexpr int NSV = 3;
    static constexpr int QBYTES = NP * NR * 128;
    static constexpr int PBYTES = KT * NR * 2;  // one P^T term: 128 keys x 32 rows, 64 bytes per key
    static constexpr int K_OFF = 0;
    static constexpr int V_OFF = K_OFF + NSK * TILE;
    static constexpr int Q_OFF = V_OFF + NSV * TILE;  // [2] query tiles
    static constexpr int P_OFF = Q_OFF + 2 * QBYTES;  // [2] buffers x (hi, lo)
    static constexpr int RED_OFF = P_OFF + 2 * 2 * PBYTES;
    static constexpr int STAT_OFF = RED_OFF + kMultiSoftmaxWarps * kMultiRPT * 4;  // [2 items][max, sum][32 rows]
    static constexpr int TAB_OFF = STAT_OFF + 2 * 2 * 32 * 4;
    // schedule tables: full-partition prefix [R + 1], remainder tiles [R], remainder order [R], counts [2],
    // then the chunks' q0, n, len, partitions [R] each
    static constexpr int TAB_INTS = 7 * kMultiLptChunks + 3;
    static constexpr int ITEM_OFF = (TAB_OFF + TAB_INTS * 4 + 15) & ~15;  // the CTA's first items, decoded
    static constexpr int BAR_OFF = ITEM_OFF + kMultiItemCache * 48;
    static constexpr int NBAR = 2 * NSK + 2 * NSV + 8 * 2 + 2 + 2;
    static constexpr int SMEM = 1024 + BAR_OFF + (NBAR + 2) * 8;
    static constexpr uint32_t TMEM_COLS = 128;
    static constexpr uint32_t S_COL = 0;   // S^T of tile t at S_COL + 32 (t & 1)
    static constexpr uint32_t O_COL = 64;  // O^T of item k at O_COL + 32 (k & 1)
    static_assert(D == 64 || D == 128, "head_dim");
    static_assert(SMEM <= 227 * 1024, "shared memory");
};

// A chunk's rows and key range as the kernel sees them: n query tokens after
// c0 = len - n prior ones; len clamped to the block table / the launch's
// partitions (flagged, as in the decode kernels).  ok = false: nothing to do
// (n <= 0 silently; an inconsistent chunk flagged when `report`).
struct MultiChunk {
    int q0, n, len, nblk, nparts;
    bool ok;
};

__device__ __forceinline__ MultiChunk multi_chunk(const MultiParams& p, int r, bool report) {
    MultiChunk c;
    c.q0 = p.query_start_loc[r];
    c.n = p.query_start_loc[r + 1] - c.q0;
    const int len_raw = p.seq_lens[r];
    c.ok = c.n > 0;
    if (c.ok && (c.n * p.group > 32 || len_raw < c.n || c.q0 < 0 || c.q0 + c.n > p.total_q_tokens)) {
        if (report) flag_error(PKV_DEVERR_LENGTH);
        c.ok = false;
    }
    c.nblk = c.ok ? decode_seq_blocks(len_raw, p.block_size, p.max_blocks_per_seq,
                                      p.num_partitions * p.partition_blocks, report)
                  : 0;
    c.len = min(len_raw, c.nblk * p.block_size);
    c.ok = c.ok && c.len >= c.n;  // a table too short for the new tokens themselves: nothing sensible to attend
    c.nparts = c.ok ? (c.nblk + p.partition_blocks - 1) / p.partition_blocks : 0;
    return c;
}

// One work item: chunk r's partition `part` for KV head g.
struct alignas(16) MultiWork {
    int r, part, g;
    int q0, n, c0, len;
    int kb, ke;  // keys [kb, ke)
    int nt;      // key tiles (0: nothing to do)
    bool direct;  // the chunk has one partition: write rows, not partials
};
static_assert(sizeof(MultiWork) == 48, "item cache entries");

// Schedule tables (longest first), built once per CTA; every thread of the
// CTA calls it (block-wide barriers), threads below num_chunks do the work.
// The chunks' geometry stays in shared memory for the items' lookups.
constexpr int kTabChunk = 3 * kMultiLptChunks + 3;  // q0, n, len, nparts: [4][kMultiLptChunks]

__device__ __forceinline__ void multi_build_schedule(const MultiParams& p, int* tab, bool report) {
    const int R = p.num_chunks;
    int* prefix = tab;                              // [R + 1]
    int* rem_tiles = tab + kMultiLptChunks + 1;     // [R]
    int* rem_order = tab + 2 * kMultiLptChunks + 1; // [R]
    int* counts = tab + 3 * kMultiLptChunks + 1;    // full items per KV head, partial chunks
    int* geo = tab + kTabChunk;
    const int t = threadIdx.x;
    const int part_tokens = p.partition_blocks * p.block_size;
    int full = 0, remt = 0;
    if (t < R) {
        const MultiChunk c = multi_chunk(p, t, report);
        if (c.ok) {
            full = c.len / part_tokens;
            const int rem = c.len - full * part_tokens;
            remt = (rem + kMultiKT - 1) / kMultiKT;
        }
        rem_tiles[t] = remt;
        prefix[t + 1] = full;
        geo[t] = c.q0;
        geo[kMultiLptChunks + t] = c.n;
        geo[2 * kMultiLptChunks + t] = c.len;
        geo[3 * kMultiLptChunks + t] = c.ok ? c.nparts : 0;
    }
    __syncthreads();
    if (t < 32) {  // inclusive scan of the full-partition counts, 32 chunks per round
        int carry = 0;
        for (int base = 0; base < R; base += 32) {
            int v = base + t < R ? prefix[base + t + 1] : 0;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int u = __shfl_up_sync(0xffffffffu, v, o);
                if (t >= o) v += u;
            }
            if (base + t < R) prefix[base + t + 1] = carry + v;
            carry += __shfl_sync(0xffffffffu, v, 31);
        }
        if (t == 0) {
            prefix[0] = 0;
            counts[0] = carry;
        }
    }
    if (t < R && remt > 0) {  // rank among the partial partitions: more tiles first, then chunk order
        int rank = 0;
        for (int q = 0; q < R; ++q) {
            const int tq = rem_tiles[q];
            rank += tq > remt || (tq == remt && q < t);
        }
        rem_order[rank] = t;
    }
    const int has = __syncthreads_count(t < R && remt > 0);  // every thread of the CTA takes part
    if (t == 0) counts[1] = has;
}

// The CTA's k-th item (rank blockIdx.x + k * gridDim.x); false past the last.
__device__ __forceinline__ bool multi_item(const MultiParams& p, const int* tab, bool lpt, int k, MultiWork& w,
                                           bool report) {
    // 32-bit ranks: the launch keeps chunks x partitions x KV heads below 2^30
    const int H = p.num_kv_heads;
    const int rank = static_cast<int>(blockIdx.x) + k * static_cast<int>(gridDim.x);
    int r, part, g;
    if (lpt) {
        const int R = p.num_chunks;
        const int* prefix = tab;
        const int* rem_order = tab + 2 * kMultiLptChunks + 1;
        const int nfull = tab[3 * kMultiLptChunks + 1] * H;
        const int nrem = tab[3 * kMultiLptChunks + 2] * H;
        if (rank < nfull) {
            const int fi = rank / H;
            g = rank - fi * H;
            int lo = 0, hi = R;  // the last chunk whose full partitions start at or before fi
            while (hi - lo > 1) {
                const int mid = (lo + hi) >> 1;
                if (prefix[mid] <= fi) lo = mid; else hi = mid;
            }
            r = lo;
            part = fi - prefix[r];
        } else if (rank < nfull + nrem) {
            const int qi = (rank - nfull) / H;
            g = (rank - nfull) - qi * H;
            r = rem_order[qi];
            part = prefix[r + 1] - prefix[r];
        } else {
            return false;
        }
    } else {
        const int per_part = p.num_chunks * H;
        if (rank >= per_part * p.num_partitions) return false;
        part = rank / per_part;
        const int rem = rank - part * per_part;
        r = rem / H;
        g = rem - r * H;
    }
    w.r = r, w.part = part, w.g = g;
    MultiChunk c;
    if (lpt) {  // the schedule reported the chunks' errors and kept their geometry
        const int* geo = tab + kTabChunk;
        c.q0 = geo[r];
        c.n = geo[kMultiLptChunks + r];
        c.len = geo[2 * kMultiLptChunks + r];
        c.nparts = geo[3 * kMultiLptChunks + r];
        c.ok = c.nparts > 0;
    } else {  // errors reported by the decoding of item (0, 0)
        c = multi_chunk(p, r, report && part == 0 && g == 0);
    }
    w.nt = 0;
    if (!c.ok || part >= c.nparts) return true;
    w.q0 = c.q0, w.n = c.n, w.len = c.len, w.c0 = c.len - c.n;
    w.kb = part * p.partition_blocks * p.block_size;
    w.ke = min(c.len, w.kb + p.partition_blocks * p.block_size);
    w.nt = (w.ke - w.kb + kMultiKT - 1) / kMultiKT;
    w.direct = c.nparts == 1;
    return true;
}

// OR of a predicate over the softmax threads (named barrier 1).
__device__ __forceinline__ bool multi_vote_any(bool v) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred q, p;\n\t"
        "setp.ne.u32 q, %1, 0;\n\t"
        "barrier.cta.red.or.pred p, 1, %2, q;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(r)
        : "r"(static_cast<uint32_t>(v)), "n"(kMultiSoftmaxThreads)
        : "memory");
    return r != 0;
}

__device__ __forceinline__ void multi_sync_softmax() {
    asm volatile("barrier.cta.sync 1, %0;" ::"n"(kMultiSoftmaxThreads) : "memory");
}

// v[c] (c < N) holds this lane's value of column c; returns the max (kMax)
// or sum over the warp's 32 lanes of column lane % N.  Each step halves the
// columns a lane keeps (N/2 + ... + 1 shuffles); the last steps join the
// lanes that kept the same column.
template <bool kMax, int N>
__device__ __forceinline__ float multi_reduce_scatter(float (&v)[N], int lane) {
#pragma unroll
    for (int o = N / 2; o >= 1; o >>= 1) {
        const bool upper = (lane & o) != 0;
#pragma unroll
        for (int j = 0; j < o; ++j) {
            const float send = upper ? v[j] : v[j + o];
            const float keep = upper ? v[j + o] : v[j];
            const float recv = __shfl_xor_sync(0xffffffffu, send, o);
            v[j] = kMax ? fmaxf(keep, recv) : keep + recv;
        }
    }
    float x = v[0];
#pragma unroll
    for (int o = N; o < 32; o <<= 1) {
        const float other = __shfl_xor_sync(0xffffffffu, x, o);
        x = kMax ? fmaxf(x, other) : x + other;
    }
    return x;
}

// N (8 or 16) consecutive 32-bit columns of this thread's TMEM lane (32x32b shape).
template <int N>
__device__ __forceinline__ void multi_tmem_ld(uint32_t taddr, float (&v)[N]) {
    uint32_t r[N];
    if constexpr (N == 16) {
        asm volatile(
            "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
            "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
            : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
              "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
            : "r"(taddr));
    } else {
        static_assert(N == 8, "columns");
        asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                     : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
                     : "r"(taddr));
    }
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < N; ++i) v[i] = __uint_as_float(r[i]);
}

template <int N>
__device__ __forceinline__ void multi_tmem_st(uint32_t taddr, const float (&v)[N]) {
    if constexpr (N == 16) {
        asm volatile(
            "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
            "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
            "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
            "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
            "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
            "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
            "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
            "r"(__float_as_uint(v[15]))
            : "memory");
    } else {
        static_assert(N == 8, "columns");
        asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(taddr),
                     "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
                     "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
                     "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7]))
                     : "memory");
    }
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

template <typename T, int D>
__global__ void __launch_bounds__(kMultiThreads, 1) paged_decode_multi_kernel(const MultiParams p, const int lpt,
                                                                            const __grid_constant__ CUtensorMap tm_q,
                                                                            const __grid_constant__ CUtensorMap tm_k,
                                                                            const __grid_constant__ CUtensorMap tm_v) {
    using C = MultiCfg<D>;
    constexpr bool kBf16 = Elem<T>::kCuType == CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    constexpr int NSK = C::NSK, NSV = C::NSV;
    constexpr int KT = kMultiKT;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align_1024(smem_raw);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF);
    uint64_t* k_full = bars;                     // [NSK] the K tile landed
    uint64_t* k_free = bars + NSK;               // [NSK] the S MMAs that read the stage are done
    uint64_t* v_full = bars + 2 * NSK;           // [NSV]
    uint64_t* v_free = bars + 2 * NSK + NSV;     // [NSV] the P.V MMAs that read the stage are done
    uint64_t* q_full = bars + 2 * NSK + 2 * NSV; // [2] per item: the Q rows landed
    uint64_t* q_free = q_full + 2;     // [2] per item: its S MMAs are done
    uint64_t* s_full = q_full + 4;     // [2] per tile: S^T(t) done
    uint64_t* s_free = q_full + 6;     // [2] per tile: the softmax read S^T(t) (256 arrivals)
    uint64_t* p_full = q_full + 8;     // [2] per tile: P^T(t) written (256 arrivals)
    uint64_t* p_free = q_full + 10;    // [2] per tile: PV(t) done
    uint64_t* o_full = q_full + 12;    // [2] per item: its last PV done
    uint64_t* o_free = q_full + 14;    // [2] per item: the epilogue read O^T and the row stats (128 arrivals)
    uint64_t* mma_done = q_full + 16;  // [2] the S / P.V issuer's MMAs are all done (exit drain)
    uint64_t* stat_full = q_full + 18; // [2] per item: the softmax wrote its rows' max and sum (256 arrivals)
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(q_full + 20);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(q_full + 21);
    int* tab = reinterpret_cast<int*>(smem + C::TAB_OFF);
    float* red = reinterpret_cast<float*>(smem + C::RED_OFF);
    float* stat = reinterpret_cast<float*>(smem + C::STAT_OFF);

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const bool lpt_order = lpt != 0;

    if (warp == 0) {
        tmem_alloc(tmem_slot, C::TMEM_COLS);
        tmem_relinquish();
    }
    if (tid == 32) {
        for (int i = 0; i < NSK; ++i) {
            mbar_init(&k_full[i], 1);
            mbar_init(&k_free[i], 1);
        }
        for (int i = 0; i < NSV; ++i) {
            mbar_init(&v_full[i], 1);
            mbar_init(&v_free[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&q_full[i], 1);
            mbar_init(&q_free[i], 1);
            mbar_init(&s_full[i], 1);
            mbar_init(&s_free[i], kMultiSoftmaxThreads);
            mbar_init(&p_full[i], kMultiSoftmaxThreads);
            mbar_init(&p_free[i], 1);
            mbar_init(&o_full[i], 1);
            mbar_init(&o_free[i], 128);
            mbar_init(&stat_full[i], kMultiSoftmaxThreads);
        }
        mbar_init(&mma_done[0], 1);
        mbar_init(&mma_done[1], 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (lpt_order) multi_build_schedule(p, tab, blockIdx.x == 0);
    // The CTA's first items, decoded once for every role (nt = -1: past the last)
    MultiWork* items = reinterpret_cast<MultiWork*>(smem + C::ITEM_OFF);
    if (lpt_order) __syncthreads();  // the schedule tables
    if (tid < kMultiItemCache) {
        MultiWork w;
        if (!multi_item(p, tab, lpt_order, tid, w, true)) w.nt = -1;
        items[tid] = w;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // item k of this CTA: false past the last one
    auto next_item = [&](int k, MultiWork& w) -> bool {
        if (k < kMultiItemCache) {
            w = items[k];
            return w.nt >= 0;
        }
        return multi_item(p, tab, lpt_order, k, w, false);
    };

    if (warp == kMultiLoadWarp || warp == kMultiLoadVWarp) {
        // ================================================================ loaders (whole warps)
        // kMultiLoadWarp: per item the Q rows, then the K tiles; kMultiLoadVWarp: the V tiles.
        // A stage is refilled as soon as the MMAs that read it are done; the
        // block ids of the next tile (across items too) are loaded one tile
        // ahead, one per lane.
        const bool k_role = warp == kMultiLoadWarp;
        const int NSR = k_role ? NSK : NSV;
        uint64_t* full = k_role ? k_full : v_full;
        uint64_t* freed = k_role ? k_free : v_free;
        const CUtensorMap* map = k_role ? &tm_k : &tm_v;
        uint8_t* ring = smem + (k_role ? C::K_OFF : C::V_OFF);
        const bool leader = lane == 0;
        const int B = p.block_size;
        const int per_tile = KT / B;  // blocks per key tile (4, 8 or 16), one lane each
        const uint64_t policy = l2_policy_evict_first();
        // a wait by lane 0, its outcome for the whole warp
        auto wait_all = [&](uint64_t* bar, int parity) -> bool {
            const int got = leader ? static_cast<int>(mbar_wait_or_abort_idle(bar, parity, abort_flag)) : 0;
            return __shfl_sync(0xffffffffu, got, 0) != 0;
        };
        auto next_work = [&](int& k, MultiWork& w) -> bool {
            while (next_item(k++, w))
                if (w.nt > 0) return true;
            return false;
        };
        auto fetch = [&](const MultiWork& w, int j) -> int {
            const int lb = w.kb / B + j * per_tile + lane;
            return (lane < per_tile && lb < (w.ke + B - 1) / B)
                       ? p.block_tables[static_cast<int64_t>(w.r) * p.max_blocks_per_seq + lb]
                       : -1;
        };
        griddep_wait();  // the pools may still be in the writes of a grid this one depends on
        int n = 0, nq = 0;  // tiles, Q tiles issued
        bool ok = true;
        int k = 0;
        MultiWork w;
        bool have = next_work(k, w);
        int ids = have ? fetch(w, 0) : -1;
        while (have && ok) {
            if (k_role) {
                const int qb = nq & 1;
                if (nq >= 2) ok = wait_all(&q_free[qb], ((nq - 2) >> 1) & 1);
                if (!ok) break;
                if (leader) {
                    // 32 / G tokens x G heads = 32 rows, token-major; rows past the
                    // chunk belong to other tokens (or are zero filled) and are masked
                    mbar_arrive_expect_tx(&q_full[qb], C::QBYTES);
#pragma unroll
                    for (int pn = 0; pn < C::NP; ++pn)
                        tma_load_3d(smem + C::Q_OFF + qb * C::QBYTES + pn * C::NR * 128, &tm_q, pn * 64,
                                    w.g * p.group, w.q0, &q_full[qb]);
                }
                ++nq;
            }
            MultiWork nw;
            bool have_next = false;
            for (int j = 0; j < w.nt; ++j) {
                int ids_next;
                if (j + 1 < w.nt) {
                    ids_next = fetch(w, j + 1);
                } else {
                    have_next = next_work(k, nw);
                    ids_next = have_next ? fetch(nw, 0) : -1;
                }
                const int lb = w.kb / B + j * per_tile + lane;
                int id = ids;
                if (lane < per_tile && lb < (w.ke + B - 1) / B && (id < 0 || id >= p.num_blocks)) {
                    flag_error(PKV_DEVERR_BLOCK_ID);
                    id = -1;
                }
                const int coord = id >= 0 ? id : static_cast<int>(p.num_blocks);  // out of range: zero fill
                const int st = n % NSR;
                if (n >= NSR) ok = wait_all(&freed[st], ((n - NSR) / NSR) & 1);
                if (!ok) break;
                if (leader) mbar_arrive_expect_tx(&full[st], C::TILE);
                __syncwarp();
                if (lane < per_tile) {
#pragma unroll
                    for (int pn = 0; pn < C::NP; ++pn)
                        tma_load_4d_hint(ring + st * C::TILE + pn * KT * 128 + lane * B * 128, map, pn * 64, w.g, 0,
                                         coord, &full[st], policy);
                }
                ++n;
                ids = ids_next;
            }
            w = nw;
            have = have_next;
        }
        if (leader) {
            // Wait (bounded) for this warp's last copies: on the normal path
            // their consumers waited for them already; after an abort they may
            // still be in flight and must land before the CTA exits.
            for (int t = max(0, nq - 2); t < nq; ++t) mbar_wait(&q_full[t & 1], (t >> 1) & 1);
            for (int t = max(0, n - NSR); t < n; ++t) mbar_wait(&full[t % NSR], (t / NSR) & 1);
        }
    } else if (warp == kMultiMmaSWarp || warp == kMultiMmaPVWarp) {
        // ================================================================ MMA issue (lane 0 of two warps)
        // The S^T and P.V streams share no accumulator or operand buffer, so
        // two threads issue them: the tensor cores take an N = 32 MMA in a
        // fraction of the time one thread needs to issue the next.
        if (lane == 0) {
            const bool s_role = warp == kMultiMmaSWarp;
            constexpr uint32_t IDESC_S = umma_idesc_f16(128, C::NR, kBf16, false, false);
            constexpr uint32_t IDESC_O = umma_idesc_f16(128, C::NR, kBf16, true, true);  // A (V^T), B (P^T) MN-major
            constexpr int kKP = KT * 128 / 16;    // panel stride of a K tile (16-byte units)
            constexpr int kQP = C::NR * 128 / 16;  // panel stride of the Q rows
            // Descriptors made once; a 16-element k slice adds its byte offset / 16.
            // V^T: M = head_dim in 64-element atoms (the tile's panels, LBO apart;
            // one panel at head_dim 64, read twice: lanes 64-127 of O^T repeat 0-63),
            // K = keys, 8 key rows per 1024-byte swizzle atom (SBO).
            const uint64_t kdesc0 = smem_desc_sw128(smem_u32(smem + C::K_OFF), 16, 1024);
            const uint64_t vdesc0 = smem_desc_sw128(smem_u32(smem + C::V_OFF), C::NP > 1 ? KT * 128 : 0, 1024);
            const uint64_t qdesc0 = smem_desc_sw128(smem_u32(smem + C::Q_OFF), 16, 1024);
            // P^T: N = 32 rows = one 64-byte swizzle atom wide (MN-major), K = keys,
            // 8 keys per 512-byte atom (SBO)
            const uint64_t pdesc0 = smem_desc_sw64(smem_u32(smem + C::P_OFF), C::PBYTES, 512);
            int it = 0, tb = 0;  // items and key tiles of this CTA so far
            bool ok = true;
            for (int k = 0; ok; ++k) {
                MultiWork w;
                if (!next_item(k, w)) break;
                if (w.nt == 0) continue;
                if (s_role) {
                    // S^T(t) = K_t . Q^T into S buffer t & 1
                    const int qb = it & 1;
                    ok = mbar_wait_or_abort_idle(&q_full[qb], (it >> 1) & 1, abort_flag);
                    const uint64_t qd = qdesc0 + qb * (C::QBYTES / 16);
                    for (int j = 0; ok && j < w.nt; ++j) {
                        const int t = tb + j;
                        ok = mbar_wait_or_abort_idle(&k_full[t % NSK], (t / NSK) & 1, abort_flag) &&
                             (t < 2 || mbar_wait_or_abort_idle(&s_free[t & 1], ((t - 2) >> 1) & 1, abort_flag));
                        if (!ok) break;
                        tc_fence_after();
                        const uint64_t kd = kdesc0 + (t % NSK) * (C::TILE / 16);
                        const uint32_t s_col = tmem + C::S_COL + 32 * (t & 1);
#pragma unroll
                        for (int kk = 0; kk < D / 16; ++kk)
                            umma_f16_ss(s_col, kd + (kk / 4) * kKP + (kk % 4) * 2, qd + (kk / 4) * kQP + (kk % 4) * 2,
                                        IDESC_S, kk > 0 ? 1u : 0u);
                        umma_commit(&s_full[t & 1]);
                        umma_commit(&k_free[t % NSK]);
                        if (j == w.nt - 1) umma_commit(&q_free[qb]);
                    }
                } else {
                    // O^T(item) += V_t^T . P_t^T; the item's first tile starts the accumulator
                    const int ob = it & 1;
                    const uint32_t o_col = tmem + C::O_COL + 32 * ob;
                    for (int j = 0; ok && j < w.nt; ++j) {
                        const int t = tb + j;
                        ok = mbar_wait_or_abort_idle(&v_full[t % NSV], (t / NSV) & 1, abort_flag) &&
                             mbar_wait_or_abort_idle(&p_full[t & 1], (t >> 1) & 1, abort_flag) &&
                             (j > 0 || it < 2 || mbar_wait_or_abort_idle(&o_free[ob], ((it - 2) >> 1) & 1, abort_flag));
                        if (!ok) break;
                        tc_fence_after();
                        const uint64_t vd = vdesc0 + (t % NSV) * (C::TILE / 16);
                        const uint64_t pd = pdesc0 + (t & 1) * (2 * C::PBYTES / 16);
#pragma unroll
                        for (int kk = 0; kk < KT / 16; ++kk) {
                            const uint64_t a = vd + kk * (16 * 128 / 16);  // 16 key rows of 128 bytes
                            const uint64_t b = pd + kk * (2 * 512 / 16);  // 16 keys: two 512-byte atoms
                            umma_f16_ss(o_col, a, b, IDESC_O, (j == 0 && kk == 0) ? 0u : 1u);
                            if constexpr (kBf16) umma_f16_ss(o_col, a, b + C::PBYTES / 16, IDESC_O, 1u);
                        }
                        umma_commit(&p_free[t & 1]);
                        umma_commit(&v_free[t % NSV]);
                        if (j == w.nt - 1) umma_commit(&o_full[ob]);
                    }
                }
                tb += w.nt;
                ++it;
            }
            // Wait (bounded) for every MMA this thread issued before tensor
            // memory is released: complete already on the normal path, possibly
            // in flight after an abort.
            uint64_t* done = &mma_done[s_role ? 0 : 1];
            umma_commit(done);
            mbar_wait(done, 0);
        }
    } else if (warp >= kMultiEpiWarp0) {
        // ================================================================ epilogue: thread t = O^T lane t
        // Once the item's last P.V is done and the softmax handed over the
        // row statistics: O^T's lane t (head_dim element t of every row) to
        // registers, O^T and the stats released, then element t of each row
        // (or of the partition's fp32 partial, and the row's max / sum).
        const int q4 = warp & 3;
        const int t = q4 * 32 + lane;
        const uint32_t lane_base = static_cast<uint32_t>(q4 * 32) << 16;
        const int G = p.group;
        int it = 0;
        bool ok = true;
        for (int k = 0; ok; ++k) {
            MultiWork w;
            if (!next_item(k, w)) break;
            if (w.nt == 0) continue;
            const int ob = it & 1;
            const int got = lane == 0 ? (mbar_wait_or_abort_idle(&o_full[ob], (it >> 1) & 1, abort_flag) &&
                                         mbar_wait_or_abort_idle(&stat_full[ob], (it >> 1) & 1, abort_flag))
                                      : 0;
            ok = __shfl_sync(0xffffffffu, got, 0) != 0;
            if (!ok) break;
            tc_fence_after();
            const float mrow = stat[ob * 64 + lane];  // row `lane`
            const float lsum = stat[ob * 64 + 32 + lane];
            const float inv = lsum > 0.f ? 1.f / lsum : 0.f;  // a row without keys writes 0
            const int R = w.n * G;
            if (!w.direct && q4 == 0 && lane < R) {
                const int64_t pi = (static_cast<int64_t>(w.q0 + lane / G) * p.num_q_heads +
                                    static_cast<int64_t>(w.g) * G + lane % G) * p.num_partitions + w.part;
                p.ws_max[pi] = mrow;
                p.ws_sum[pi] = lsum;
            }
            // O^T's lane t in two halves of 16 rows (lanes past head_dim 64 repeat
            // 0-63); O^T and the stats are released once both are out: the next
            // item on this O^T buffer is two items away
            if (q4 * 32 < D) {
                // row r = i G + hh: element t sits (i Hq + hh) rows (times the
                // partitions for partials) after the item's first row
                const int64_t row0 = static_cast<int64_t>(w.q0) * p.num_q_heads + static_cast<int64_t>(w.g) * G;
                T* out_t = reinterpret_cast<T*>(p.out) + row0 * D + t;
                float* part_t = w.direct ? nullptr : p.ws_out + (row0 * p.num_partitions + w.part) * D + t;
                const int row_step = w.direct ? D : p.num_partitions * D;   // next head
                const int tok_step = (p.num_q_heads - G) * row_step;        // next token, after G heads
                int off = 0, hh = 0;
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    float o[16];
                    multi_tmem_ld<16>(tmem + lane_base + C::O_COL + 32 * ob + 16 * half, o);
#pragma unroll
                    for (int c = 0; c < 16; ++c) {
                        const int r = 16 * half + c;
                        const float val = o[c] * __shfl_sync(0xffffffffu, inv, r);
                        if (r < R) {
                            if (w.direct)
                                out_t[off] = Elem<T>::from_f(val);
                            else
                                part_t[off] = val;
                        }
                        off += row_step;
                        if (++hh == G) hh = 0, off += tok_step;
                    }
                }
            }
            tc_fence_before();
            mbar_arrive(&o_free[ob]);
            ++it;
        }
    } else {
        // ================================================================ softmax
        // Thread (quadrant q = warp % 4, lane): TMEM lane t = 32 q + lane, i.e.
        // key t of the tile for S^T and head_dim element t for O^T; the warp
        // group h = warp / 4 takes rows (columns) RPT h .. RPT h + RPT - 1.
        constexpr int RPT = kMultiRPT;
        const int q4 = warp & 3, h = warp >> 2;
        const int t = q4 * 32 + lane;
        const int c0r = RPT * h;  // first row of this thread
        const uint32_t lane_base = static_cast<uint32_t>(q4 * 32) << 16;
        const int G = p.group;
        const int B = p.block_size;
        const float sl2 = p.scale_log2;
        // Lazy rescaling: a row's exponent base m moves (and O^T and the sums
        // are rescaled) only when some score exceeds it by more than 2^8; the
        // weights exp2(s - m) then stay below 256, inside the 16-bit P range.
        constexpr float kRescaleLog2 = 8.f;
        int it = 0, tb = 0;
        bool ok = true;
        for (int k = 0;; ++k) {
            MultiWork w;
            if (!next_item(k, w)) break;
            if (w.nt == 0) continue;
            const int R = w.n * G;
            const bool active = c0r < R;  // this row group holds rows of the chunk
            const uint32_t to = tmem + lane_base + C::O_COL + 32 * (it & 1) + c0r;
            // mb: the rows' exponent bases (log2 domain), set by the item's first
            // tile (which always votes for new bases); l: this thread's partial
            // row sums.  A row past the chunk's rows keeps mb = +inf: its
            // weights are 0 and it never votes.  A row without a key yet keeps
            // base 0 (its sum and O^T column are 0).
            float mb[RPT], l[RPT];
#pragma unroll
            for (int c = 0; c < RPT; ++c) {
                mb[c] = c0r + c < R ? 0.f : INFINITY;
                l[c] = 0.f;
            }
            // keys past the context in its last block (the chunk's last
            // partition only): their V rows may hold anything, and 0 * NaN must
            // not reach O^T, so they are zeroed before P.V
            const int dead_lo = w.len;
            const int dead_hi = w.ke == w.len ? ((w.len + B - 1) / B) * B : w.len;
            for (int j = 0; j < w.nt; ++j) {
                const int tt = tb + j;
                const int sb = tt & 1;
                ok = ok && mbar_wait_or_abort(&s_full[sb], (tt >> 1) & 1, abort_flag);
                tc_fence_after();
                float s[RPT];
                if (active) multi_tmem_ld<RPT>(tmem + lane_base + C::S_COL + 32 * sb + c0r, s);
                tc_fence_before();
                mbar_arrive(&s_free[sb]);
                // ---- mask: row r = i G + hh sees key pos iff pos <= c0 + i, i < n, pos < ke;
                // a tile whose keys all lie before the chunk's first new token and
                // inside the partition needs none
                const int pos = w.kb + j * KT + t;
                const int tk0 = w.kb + j * KT;
                bool exceed = false;
                if (active) {
                    if (tk0 + KT - 1 <= min(w.c0, w.ke - 1)) {
#pragma unroll
                        for (int c = 0; c < RPT; ++c) {
                            s[c] *= sl2;
                            exceed |= s[c] > mb[c] + kRescaleLog2;
                        }
                    } else {
                        const int rlo = (pos >= w.ke ? C::NR : (pos <= w.c0 ? 0 : (pos - w.c0) * G)) - c0r;
#pragma unroll
                        for (int c = 0; c < RPT; ++c) {
                            s[c] = c >= rlo ? s[c] * sl2 : -INFINITY;
                            exceed |= s[c] > mb[c] + kRescaleLog2;
                        }
                    }
                }
                // ---- one vote per tile: a wait gave up, or a row's base must move.
                // Then every softmax thread leaves together, or the tile's row
                // maxima over its 128 keys become the new bases.
                if (multi_vote_any(exceed || j == 0 || !ok)) {
                    if (multi_vote_any(!ok)) {
                        ok = false;
                        break;
                    }
                    if (active) {
                        float v[RPT];
#pragma unroll
                        for (int c = 0; c < RPT; ++c) v[c] = s[c];
                        const float wm = multi_reduce_scatter<true, RPT>(v, lane);  // column lane % RPT over this warp's keys
                        if (lane < RPT) red[warp * RPT + lane] = wm;
                    }
                    multi_sync_softmax();
                    if (active) {
                        const int cc = lane % RPT;
                        const float cm = fmaxf(fmaxf(red[(4 * h + 0) * RPT + cc], red[(4 * h + 1) * RPT + cc]),
                                               fmaxf(red[(4 * h + 2) * RPT + cc], red[(4 * h + 3) * RPT + cc]));
                        bool moved = false;  // the same on the threads of a row group: m and cm are
#pragma unroll
                        for (int c = 0; c < RPT; ++c) moved |= __shfl_sync(0xffffffffu, cm, c) > mb[c];
                        // O^T *= alpha once the previous P.V is done (the next one waits
                        // for this tile's P); on an item's first tile O^T is not started
                        const bool rescale_o = j > 0 && moved;
                        if (rescale_o)
                            ok = __all_sync(0xffffffffu,
                                            ok && mbar_wait_or_abort(&p_free[(tt - 1) & 1], ((tt - 1) >> 1) & 1, abort_flag));
                        float o[RPT];
                        if (rescale_o && ok) {
                            tc_fence_after();
                            multi_tmem_ld<RPT>(to, o);
                        }
#pragma unroll
                        for (int c = 0; c < RPT; ++c) {
                            // the first tile starts the bases; a row past the chunk stays at +inf
                            const float old = j == 0 && mb[c] != INFINITY ? -INFINITY : mb[c];
                            float mn = fmaxf(old, __shfl_sync(0xffffffffu, cm, c));
                            mn = mn == -INFINITY ? 0.f : mn;  // no key yet
                            const float alpha = j == 0 || mn == mb[c] ? 1.f : ex2_approx(mb[c] - mn);
                            mb[c] = mn;
                            l[c] *= alpha;
                            o[c] *= alpha;
                        }
                        if (rescale_o && ok) multi_tmem_st<RPT>(to, o);
                    }
                }
                // ---- P^T(r, key t) = exp2(s - m), bf16 as hi + lo (hi: the top 16
                // bits of P; lo: the exact remainder rounded, |lo| < 2^-7 |P|).  A
                // row group past the chunk's rows skips it: P.V then mixes stale
                // P^T rows into O^T columns that are never read.
                if (active) {
#pragma unroll
                    for (int c = 0; c < RPT; ++c) {
                        s[c] = ex2_approx(s[c] - mb[c]);  // the weights, in place
                        l[c] += s[c];
                    }
                }
                if (active && tt >= 2)
                    ok = __all_sync(0xffffffffu, ok && mbar_wait_or_abort(&p_free[sb], ((tt - 2) >> 1) & 1, abort_flag));
                if (active && ok) {
                    // P^T is the B operand in the MN-major, 64-byte-swizzled layout:
                    // key k's 32 row weights are 64 contiguous bytes (k % 8 of an
                    // 8-key, 512-byte atom; 16-byte piece q at q ^ ((k >> 1) & 3)),
                    // so this thread's rows are 16-byte pieces of one line.
                    uint8_t* line = smem + C::P_OFF + sb * 2 * C::PBYTES + (t >> 3) * 512 + (t & 7) * 64;
                    const int sw = (t >> 1) & 3;
#pragma unroll
                    for (int q = 0; q < RPT / 8; ++q) {
                        uint8_t* dst = line + ((((c0r >> 3) + q) ^ sw) << 4);
                        uint32_t hw[4], lw[4];
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const float a = s[8 * q + 2 * i], b = s[8 * q + 2 * i + 1];
                            if constexpr (kBf16) {
                                const uint32_t ba = __float_as_uint(a), bb = __float_as_uint(b);
                                hw[i] = __byte_perm(ba, bb, 0x7632);  // the top 16 bits of each
                                lw[i] = Elem<T>::pack(a - __uint_as_float(ba & 0xFFFF0000u),
                                                      b - __uint_as_float(bb & 0xFFFF0000u));
                            } else {
                                hw[i] = Elem<T>::pack(a, b);
                            }
                        }
                        *reinterpret_cast<uint4*>(dst) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
                        if constexpr (kBf16)
                            *reinterpret_cast<uint4*>(dst + C::PBYTES) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
                    }
                }
                // ---- dead V rows of this tile (the row group h = 0 threads zero them)
                if (h == 0 && dead_lo < dead_hi && dead_hi > tk0 && dead_lo < tk0 + KT) {
                    ok = __all_sync(0xffffffffu, ok && mbar_wait_or_abort(&v_full[tt % NSV], (tt / NSV) & 1, abort_flag));
                    if (ok && pos >= dead_lo && pos < dead_hi) {
                        uint8_t* vrow = smem + C::V_OFF + (tt % NSV) * C::TILE + t * 128;
#pragma unroll
                        for (int pn = 0; pn < C::NP; ++pn)
#pragma unroll
                            for (int cq = 0; cq < 8; ++cq)
                                *reinterpret_cast<uint4*>(vrow + pn * KT * 128 + cq * 16) = make_uint4(0, 0, 0, 0);
                    }
                }
                if (active) fence_proxy_async();  // P^T and zeroed V rows -> the tensor cores' (async) proxy
                tc_fence_before();
                mbar_arrive(&p_full[sb]);
            }
            // ---- hand the item over to the epilogue warps: each row's exponent
            // base and sum (the rows themselves stay in O^T)
            if (multi_vote_any(!ok)) {
                ok = false;
                break;
            }
            {
                float v[RPT];
#pragma unroll
                for (int c = 0; c < RPT; ++c) v[c] = l[c];
                const float ws = multi_reduce_scatter<false, RPT>(v, lane);
                if (lane < RPT) red[warp * RPT + lane] = ws;
            }
            multi_sync_softmax();
            {
                const int cc = lane % RPT;
                const float cl = (red[(4 * h + 0) * RPT + cc] + red[(4 * h + 1) * RPT + cc]) +
                                 (red[(4 * h + 2) * RPT + cc] + red[(4 * h + 3) * RPT + cc]);
                // the slot of item it - 2 is free once its epilogue read it
                if (it >= 2) ok = ok && mbar_wait_or_abort(&o_free[it & 1], ((it - 2) >> 1) & 1, abort_flag);
                float* st_m = stat + (it & 1) * 64;
                if (q4 == 0 && ok) {
                    if (lane < RPT) st_m[32 + c0r + lane] = cl;
                    if (lane == 0) {
#pragma unroll
                        for (int c = 0; c < RPT; ++c) st_m[c0r + c] = mb[c];
                    }
                }
                mbar_arrive(&stat_full[it & 1]);
            }
            tb += w.nt;
            ++it;
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

// ---- merge of the partitions of multi-token rows: one warp per (row, q head).
struct MultiMergeParams {
    void* out;
    const int32_t* seq_lens;
    const int32_t* query_start_loc;
    const float* ws_max;
    const float* ws_sum;
    const float* ws_out;
    int num_chunks;
    int num_q_heads;
    int64_t total_q_tokens;
    int block_size;
    int max_blocks_per_seq;
    int partition_blocks;
    int num_partitions;
};

template <typename T, int D>
__global__ void __launch_bounds__(128) paged_decode_multi_merge_kernel(const MultiMergeParams p) {
    const int64_t wid = static_cast<int64_t>(blockIdx.x) * 4 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (wid >= p.total_q_tokens * p.num_q_heads) return;
    const int64_t row = wid / p.num_q_heads;
    // the chunk that owns this row: the last r with query_start_loc[r] <= row
    int lo = 0, hi = p.num_chunks;  // invariant: qsl[lo] <= row < qsl[hi] (when row is covered)
    if (row < p.query_start_loc[0] || row >= p.query_start_loc[p.num_chunks]) return;
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (p.query_start_loc[mid] <= row) lo = mid; else hi = mid;
    }
    const int nblk = decode_seq_blocks(p.seq_lens[lo], p.block_size, p.max_blocks_per_seq,
                                       p.num_partitions * p.partition_blocks, false);
    const int nparts = nblk > 0 ? (nblk + p.partition_blocks - 1) / p.partition_blocks : 1;
    if (nparts <= 1) return;  // the attention kernel wrote this row itself
    griddep_wait();           // the partials are the writes of the attention grid
    const float* pm = p.ws_max + wid * p.num_partitions;
    const float* pl = p.ws_sum + wid * p.num_partitions;
    const float* po = p.ws_out + wid * p.num_partitions * D;
    float mx = -INFINITY;
    for (int i = lane; i < nparts; i += 32) mx = fmaxf(mx, pm[i]);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    float wsum = 0.f;
    for (int i = lane; i < nparts; i += 32) wsum += pm[i] == -INFINITY ? 0.f : pl[i] * exp2f(pm[i] - mx);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) wsum += __shfl_xor_sync(0xffffffffu, wsum, off);
    constexpr int DPL = D / 32;
    float o[DPL];
#pragma unroll
    for (int j = 0; j < DPL; ++j) o[j] = 0.f;
    for (int i = 0; i < nparts; ++i) {
        const float w = pm[i] == -INFINITY ? 0.f : pl[i] * exp2f(pm[i] - mx);
        const float* src = po + static_cast<int64_t>(i) * D + lane * DPL;
#pragma unroll
        for (int j = 0; j < DPL; ++j) o[j] = fmaf(w, src[j], o[j]);
    }
    const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
    T* dst = reinterpret_cast<T*>(p.out) + wid * D + lane * DPL;
#pragma unroll
    for (int j = 0; j < DPL; ++j) dst[j] = Elem<T>::from_f(o[j] * inv);
}


}  // namespace pkv
