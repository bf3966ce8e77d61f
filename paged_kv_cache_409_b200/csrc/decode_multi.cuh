// decode_multi.cuh -- multi-token decode: each sequence (a "chunk") holds n
// new tokens at the end of its context (speculative verification of n draft
// tokens, guide page "Speculative Decoding": a small draft model proposes the
// next tokens and the large model checks them all in one pass).  Row i of a
// chunk with c0 = seq_len - n prior tokens attends causally to keys
// j <= c0 + i -- the chunked-prefill definition, for chunks of a few tokens.
//
// With n * G query rows per KV head (G query heads share one), the work per
// K/V byte is 4 * n * G flops: too little for tcgen05's 128-row tiles (the
// prefill kernel spends its time in the per-tile softmax of 128 rows of which
// n * G are live) and too much for the CUDA cores.  The rows therefore go to
// the M side of warp MMAs (mma.sync m16n8k16, fp32 accumulation), 16 rows per
// warp, in the usual register layout of attention kernels on warp MMAs:
//   S [16 rows x 16 keys]  = Q [16 x D] . K^T       (B: ldmatrix of the K tile)
//   O [16 rows x D]       += P [16 x 16 keys] . V   (A: S accumulators reused,
//                                                     B: ldmatrix.trans of V)
// Rows are (token, head) pairs, token-major: row r = i * G + hh.  A CTA serves
// one (chunk, partition, KV head); its warps form one row group of 16 rows per
// 16 live rows (at most RG) and NW / groups streams, each warp with its own
// TMA pipeline over the 16-token units (sub-blocks) of its stream, and its own
// online-softmax state.  Warps of
// one row group merge in shared memory; the CTA writes output rows (one
// partition) or partials for the merge kernel, which combines partitions as
// the decode merge does.
#pragma once

#include "decode.cuh"

namespace pkv {

struct MultiParams {
    void* out;                       // [total_q_tokens, Hq, D]
    const void* query;               // [total_q_tokens, Hq, D]
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
    int max_blocks_per_seq;
    int64_t num_blocks;
    int partition_blocks;
    int num_partitions;
    int64_t total_q_tokens;
};

template <typename T, int D, int B, int NST, int NW, int RG>
struct MultiCfg {
    static constexpr int TB = 2;
    static constexpr int UT = B < 16 ? B : 16;        // tokens per unit (one TMA stage)
    static constexpr int UPB = B / UT;                // units per block
    static constexpr int NP = D * TB / 128;           // 128-byte panels per row
    static constexpr int TILE = UT * D * TB;          // one unit of K (or V) for one KV head
    static constexpr int STAGE = 2 * TILE;
    static constexpr int STAGES_BYTES = NW * NST * STAGE;
    static constexpr int RED_BYTES = NW * 16 * (D + 2) * 4;
    static constexpr int BT_OFF = STAGES_BYTES > RED_BYTES ? STAGES_BYTES : RED_BYTES;
    static_assert(TILE % 1024 == 0, "tiles must keep 1024-byte alignment for the 128-byte swizzle");
    static_assert(NW % RG == 0, "warps must split evenly into row groups");
    // per warp: NST full barriers, then NST empty barriers (used when two row groups share a stream's stages)
    static size_t smem_bytes(int pb) { return 1024 + BT_OFF + static_cast<size_t>(pb) * 4 + 16 + 2 * NW * NST * 8; }
};

// Resident CTAs per SM the register allocation must allow (launch bounds):
// three 4-warp CTAs (168 registers) -- left free, the compiler takes 203 and
// two CTAs fit, 10 % slower on the multi-token batch; a fourth CTA (128
// registers) spills and is slower still.
#ifndef PKV_MULTI_MIN_CTAS
#define PKV_MULTI_MIN_CTAS 3
#endif

template <typename T, int D, int B, int NST, int NW, int RG>
__global__ void __launch_bounds__(NW * 32, PKV_MULTI_MIN_CTAS) paged_decode_multi_kernel(const MultiParams p, const int G,
                                                                     const __grid_constant__ CUtensorMap tm_k,
                                                                     const __grid_constant__ CUtensorMap tm_v) {
    using C = MultiCfg<T, D, B, NST, NW, RG>;
    constexpr bool kBf16 = Elem<T>::kCuType == CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    constexpr int KS = D / 16;  // 16-dim steps of Q.K^T
    constexpr int DT = D / 8;   // 8-dim output tiles
    constexpr int UT = C::UT;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align_1024(smem_raw);

    const int per_chunk = p.num_partitions * p.num_kv_heads;
    const int r = blockIdx.x / per_chunk;
    const int rem = blockIdx.x - r * per_chunk;
    const int part = rem / p.num_kv_heads;
    const int g = rem - part * p.num_kv_heads;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    const int q0 = p.query_start_loc[r];
    const int n = p.query_start_loc[r + 1] - q0;
    const int len_raw = p.seq_lens[r];
    if (n <= 0) return;
    if (n * G > 16 * RG || len_raw < n || q0 < 0 || q0 + n > p.total_q_tokens) {
        if (threadIdx.x == 0 && part == 0 && g == 0) flag_error(PKV_DEVERR_LENGTH);
        return;
    }
    const int nblk = decode_seq_blocks(len_raw, B, p.max_blocks_per_seq, p.num_partitions * p.partition_blocks,
                                       threadIdx.x == 0 && part == 0 && g == 0);
    const int len = min(len_raw, nblk * B);
    const int c0 = len - n;  // a clamped sequence keeps its last rows' limits inside the table
    const int nparts = nblk > 0 ? (nblk + p.partition_blocks - 1) / p.partition_blocks : 1;
    if (part >= nparts) return;
    const int b0 = part * p.partition_blocks;
    const int nb = max(0, min(nblk - b0, p.partition_blocks));
    const bool direct = nparts == 1;

    int* bt_s = reinterpret_cast<int*>(smem + C::BT_OFF);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + ((C::BT_OFF + p.partition_blocks * 4 + 15) & ~15));
    const int32_t* bt_row = p.block_tables + static_cast<int64_t>(r) * p.max_blocks_per_seq + b0;
    for (int i = threadIdx.x; i < nb; i += NW * 32) {
        int id = bt_row[i];
        if (id < 0 || id >= p.num_blocks) {
            flag_error(PKV_DEVERR_BLOCK_ID);
            id = -1;
        }
        bt_s[i] = id;
    }
    // ---- this warp's 16 rows: the lane holds rows rq and rq + 8 (rq = lane / 4).
    // A chunk with at most 16 rows uses one row group: every warp is a stream.
    // With two row groups the two warps of a stream share its stages: the
    // first issues each unit's copy once into a ring of 2 * NST stages, both
    // read it, and each releases it on the stage's empty barrier.
    const int nrg = n * G > 16 ? RG : 1;
    const int nsw = NW / nrg;
    const int rg = warp % nrg, stream = warp / nrg;
    const int ring = nrg * NST;
    uint64_t* fbar = bars + stream * ring;            // full: the unit's bytes arrived
    uint64_t* ebar = bars + NW * NST + stream * ring;  // empty: every reader of the stage is done
    if (lane == 0) {
#pragma unroll
        for (int st = 0; st < NST; ++st) {
            mbar_init(&bars[warp * NST + st], 1);
            mbar_init(&bars[NW * NST + warp * NST + st], nrg);
        }
        fence_mbar_init();
    }
    __syncthreads();

    // units (16-token sub-blocks) holding positions [b0 * B, min(len, (b0 + nb) * B))
    const int span = max(0, min(len, (b0 + nb) * B) - b0 * B);
    const int units = (span + UT - 1) / UT;
    const int nw = units > stream ? (units - stream + nsw - 1) / nsw : 0;
    uint8_t* wstage = smem + stream * ring * C::STAGE;  // the stream's ring of stages
    const bool producer = rg == 0;
    const uint64_t policy = l2_policy_evict_first();

    auto issue = [&](int k) {  // lane 0 of the producer only
        const int st = k % ring;
        const int u = stream + k * nsw;
        const int id = bt_s[u / C::UPB];
        const int coord = id >= 0 ? id : static_cast<int>(p.num_blocks);  // out of range: zero fill
        const int row0 = (u % C::UPB) * UT;
        uint8_t* kd = wstage + st * C::STAGE;
        uint8_t* vd = kd + C::TILE;
        mbar_arrive_expect_tx(&fbar[st], C::STAGE);
#pragma unroll
        for (int pn = 0; pn < C::NP; ++pn) {
            tma_load_4d_hint(kd + pn * UT * 128, &tm_k, pn * 64, g, row0, coord, &fbar[st], policy);
            tma_load_4d_hint(vd + pn * UT * 128, &tm_v, pn * 64, g, row0, coord, &fbar[st], policy);
        }
    };
    int issued = 0;
    griddep_wait();  // the pools may still be in the writes of a grid this one depends on
    if (lane == 0 && producer) {
        for (; issued < ring && issued < nw; ++issued) issue(issued);
    }
    __syncwarp();
    // The query fragments load while the first stages are in flight.
    const int gq = lane >> 2, cq = lane & 3;
    int lim[2];  // last key position each of the lane's two rows may see
    uint32_t qa[KS][4];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int row = 16 * rg + gq + 8 * h;
        const int i = row / G, hh = row - (row / G) * G;
        lim[h] = c0 + min(i, n - 1);
        const bool live = i < n;
        const T* qrow = reinterpret_cast<const T*>(p.query) +
                        ((static_cast<int64_t>(q0) + (live ? i : 0)) * p.num_q_heads + static_cast<int64_t>(g) * G +
                         hh) * D;
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {
            qa[ks][h] = live ? *reinterpret_cast<const uint32_t*>(qrow + 16 * ks + 2 * cq) : 0u;
            qa[ks][h + 2] = live ? *reinterpret_cast<const uint32_t*>(qrow + 16 * ks + 8 + 2 * cq) : 0u;
        }
    }

    float m[2] = {-INFINITY, -INFINITY}, l[2] = {0.f, 0.f};
    float o[DT][4];  // [dim tile j][c0: (row rq, dim 8j + 2cq), c1: +1, c2: (row rq + 8, dim 8j + 2cq), c3: +1]
#pragma unroll
    for (int j = 0; j < DT; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
    const int lr = lane & 7, lm = lane >> 3;

    int k = 0;
    for (; k < nw; ++k) {
        const int st = k % ring;
        const bool ok = mbar_wait_main(&fbar[st], (k / ring) & 1);
        if (!__all_sync(0xffffffffu, ok)) break;
        const int u = stream + k * nsw;
        const int pos0 = (b0 + u / C::UPB) * B + (u % C::UPB) * UT;  // key position of the unit's first token
        const int valid = min(UT, len - pos0);
        if (bt_s[u / C::UPB] >= 0) {
            const uint8_t* Ks = wstage + st * C::STAGE;
            const uint8_t* Vs = Ks + C::TILE;
            // ---- S = Q . K^T: s[nt] covers keys 8 nt .. 8 nt + 7 of the unit
            // two accumulator sets (even / odd dim steps) halve the dependent MMA chain
            float s[2][4], s2[2][4];
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
                s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
                s2[nt][0] = s2[nt][1] = s2[nt][2] = s2[nt][3] = 0.f;
            }
#pragma unroll
            for (int ks = 0; ks < KS; ++ks) {
                float (&acc)[2][4] = (ks & 1) ? s2 : s;
                if constexpr (UT == 16) {
                    // matrices: (keys 0-7, chunk 2ks), (keys 0-7, chunk 2ks+1), (keys 8-15, ...), (keys 8-15, ...)
                    const int key = lr + 8 * (lm >> 1);
                    const int ch = 2 * ks + (lm & 1);
                    uint32_t b[4];
                    ldsm_x4(b, Ks + (ch / 8) * UT * 128 + key * 128 + (((ch % 8) ^ (key & 7)) << 4));
                    mma_16816<kBf16>(acc[0], qa[ks], b[0], b[1]);
                    mma_16816<kBf16>(acc[1], qa[ks], b[2], b[3]);
                } else {
                    const int key = lr;
                    const int ch = 2 * ks + (lm & 1);
                    uint32_t b0r, b1r;
                    ldsm_x2(b0r, b1r, Ks + (ch / 8) * UT * 128 + key * 128 + (((ch % 8) ^ (key & 7)) << 4));
                    mma_16816<kBf16>(acc[0], qa[ks], b0r, b1r);
                }
            }
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) s[nt][e] += s2[nt][e];
            // ---- causal mask and online softmax of the lane's two rows (log2 domain)
            float bm[2] = {-INFINITY, -INFINITY};
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int key = 8 * nt + 2 * cq + (e & 1);
                    const int h = e >> 1;
                    const bool ok_key = (UT == 16 || nt == 0) && key < valid && pos0 + key <= lim[h];
                    s[nt][e] = ok_key ? s[nt][e] * p.scale_log2 : -INFINITY;
                    bm[h] = fmaxf(bm[h], s[nt][e]);
                }
            }
            // Lazy rescaling: a row's exponent base m moves, and its O and sum
            // are rescaled, only when a unit's max exceeds it by more than 2^8;
            // the weights exp2(s - m) then stay below 256 (bf16 / f16 P).
            float alpha[2] = {1.f, 1.f}, msafe[2];
            bool rs = false;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                bm[h] = fmaxf(bm[h], __shfl_xor_sync(0xffffffffu, bm[h], 1));
                bm[h] = fmaxf(bm[h], __shfl_xor_sync(0xffffffffu, bm[h], 2));
                if (bm[h] > m[h] + 8.f || (m[h] == -INFINITY && bm[h] != -INFINITY)) {
                    alpha[h] = ex2_approx(m[h] - bm[h]);  // 0 when m was -inf
                    m[h] = bm[h];
                    rs = true;
                }
                msafe[h] = m[h] == -INFINITY ? 0.f : m[h];  // a row with no key yet stays empty
            }
            float ps[2] = {0.f, 0.f};
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    s[nt][e] = ex2_approx(s[nt][e] - msafe[e >> 1]);
                    ps[e >> 1] += s[nt][e];
                }
            }
            l[0] = l[0] * alpha[0] + ps[0];  // per-lane partial row sums; the quad is summed at the end
            l[1] = l[1] * alpha[1] + ps[1];
            if (__any_sync(0xffffffffu, rs)) {
#pragma unroll
                for (int j = 0; j < DT; ++j) {
                    o[j][0] *= alpha[0];
                    o[j][1] *= alpha[0];
                    o[j][2] *= alpha[1];
                    o[j][3] *= alpha[1];
                }
            }
            // ---- O += P . V  (P: the S accumulators in the A layout; bf16 as hi + lo)
            uint32_t pa[4], pl[4] = {0u, 0u, 0u, 0u};
            pa[0] = Elem<T>::pack(s[0][0], s[0][1]);
            pa[1] = Elem<T>::pack(s[0][2], s[0][3]);
            pa[2] = Elem<T>::pack(s[1][0], s[1][1]);
            pa[3] = Elem<T>::pack(s[1][2], s[1][3]);
            if constexpr (kBf16) {
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 f = Elem<T>::pair(pa[e]);
                    pl[e] = Elem<T>::pack(s[e >> 1][2 * (e & 1)] - f.x, s[e >> 1][2 * (e & 1) + 1] - f.y);
                }
            }
            // keys of this lane's B fragment halves, for masking rows past the context
            const bool partial = valid < 16;
            const int t0 = 2 * cq;
            const uint32_t mk0 = (t0 < valid ? 0x0000FFFFu : 0u) | (t0 + 1 < valid ? 0xFFFF0000u : 0u);
            const uint32_t mk1 = (t0 + 8 < valid ? 0x0000FFFFu : 0u) | (t0 + 9 < valid ? 0xFFFF0000u : 0u);
#pragma unroll
            for (int jp = 0; jp < DT / 2; ++jp) {
                uint32_t b[4];
                if constexpr (UT == 16) {
                    // matrices: (keys 0-7, chunk 2jp), (keys 8-15, chunk 2jp), (keys 0-7, 2jp+1), (keys 8-15, 2jp+1)
                    const int key = lr + 8 * (lm & 1);
                    const int ch = 2 * jp + (lm >> 1);
                    ldsm_x4_trans(b, Vs + (ch / 8) * UT * 128 + key * 128 + (((ch % 8) ^ (key & 7)) << 4));
                } else {
                    const int key = lr;
                    const int ch = 2 * jp + (lm & 1);
                    ldsm_x2_trans(b[0], b[2], Vs + (ch / 8) * UT * 128 + key * 128 + (((ch % 8) ^ (key & 7)) << 4));
                    b[1] = b[3] = 0u;
                }
                if (partial) {  // rows past the context may hold anything: 0 * NaN must not reach O
                    b[0] &= mk0;
                    b[2] &= mk0;
                    b[1] &= mk1;
                    b[3] &= mk1;
                }
                mma_16816<kBf16>(o[2 * jp], pa, b[0], b[1]);
                mma_16816<kBf16>(o[2 * jp + 1], pa, b[2], b[3]);
                if constexpr (kBf16) {
                    mma_16816<kBf16>(o[2 * jp], pl, b[0], b[1]);
                    mma_16816<kBf16>(o[2 * jp + 1], pl, b[2], b[3]);
                }
            }
        }
        __syncwarp();
        bool go = true;
        if (lane == 0) {
            if (nrg > 1) mbar_arrive(&ebar[st]);
            if (producer && k + ring < nw) {
                // the stage is refilled once every reader released unit k
                go = nrg == 1 || mbar_wait_main(&ebar[st], (k / ring) & 1);
                if (go) {
                    fence_proxy_async();
                    issue(k + ring);
                    issued = k + ring + 1;
                }
            }
        }
        if (!__shfl_sync(0xffffffffu, go, 0)) {
            ++k;
            break;
        }
    }
    if (k < nw && lane == 0 && producer) {
        // a wait gave up: wait (bounded) for this warp's copies still in flight
        for (int kk = k; kk < issued; ++kk) mbar_wait(&fbar[kk % ring], (kk / ring) & 1);
    }
    if (k < nw) m[0] = m[1] = -INFINITY, l[0] = l[1] = 0.f;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        l[h] += __shfl_xor_sync(0xffffffffu, l[h], 1);
        l[h] += __shfl_xor_sync(0xffffffffu, l[h], 2);
    }

    // ---- merge the streams of each row group, write rows or partials
    __syncthreads();
    float* red_m = reinterpret_cast<float*>(smem);  // [NW][16]
    float* red_l = red_m + NW * 16;                 // [NW][16]
    float* red_o = red_l + NW * 16;                 // [NW][16][D]
    if (cq == 0) {
        red_m[warp * 16 + gq] = m[0], red_l[warp * 16 + gq] = l[0];
        red_m[warp * 16 + gq + 8] = m[1], red_l[warp * 16 + gq + 8] = l[1];
    }
#pragma unroll
    for (int j = 0; j < DT; ++j) {
        const int d = 8 * j + 2 * cq;
        *reinterpret_cast<float2*>(&red_o[(warp * 16 + gq) * D + d]) = make_float2(o[j][0], o[j][1]);
        *reinterpret_cast<float2*>(&red_o[(warp * 16 + gq + 8) * D + d]) = make_float2(o[j][2], o[j][3]);
    }
    __syncthreads();
    const int rows = n * G;
    for (int idx = threadIdx.x; idx < rows * D; idx += NW * 32) {
        const int row = idx / D, d = idx - row * D;
        const int rgr = row / 16, rr = row - rgr * 16;
        float mx = -INFINITY;
        for (int w = rgr; w < NW; w += nrg) mx = fmaxf(mx, red_m[w * 16 + rr]);
        float sum = 0.f, acc = 0.f;
        if (mx != -INFINITY) {
            for (int w = rgr; w < NW; w += nrg) {
                const float mw = red_m[w * 16 + rr];
                if (mw != -INFINITY) {
                    const float f = exp2f(mw - mx);
                    sum += red_l[w * 16 + rr] * f;
                    acc += red_o[(w * 16 + rr) * D + d] * f;
                }
            }
        }
        const float val = mx != -INFINITY ? acc / sum : 0.f;
        const int i = row / G, hh = row - (row / G) * G;
        const int64_t orow = (static_cast<int64_t>(q0) + i) * p.num_q_heads + static_cast<int64_t>(g) * G + hh;
        if (direct) {
            reinterpret_cast<T*>(p.out)[orow * D + d] = Elem<T>::from_f(val);
        } else {
            const int64_t pi = orow * p.num_partitions + part;
            p.ws_out[pi * D + d] = val;
            if (d == 0) {
                p.ws_max[pi] = mx;
                p.ws_sum[pi] = sum;
            }
        }
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
