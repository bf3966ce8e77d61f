// decode.cuh -- paged decode attention (one query token per sequence) and the
// log-sum-exp merge of split-K partitions.
//
// Decode is a streaming, HBM-bound kernel: each K/V byte of a sequence's
// context is read once per KV head, and all G query heads that share that KV
// head (grouped-query attention) are served from the same bytes.
//
// The kernel below computes on the CUDA cores and serves fp32 pools; fp16 and
// bf16 pools use the tensor-core variant in decode_mma.cuh, which shares the
// parameters, the partitioning, the merge and decode_finish defined here.
//
// Work decomposition: one CTA per (sequence, partition, KV head), KV head
// fastest so that CTAs running together read neighbouring bytes of the same
// physical blocks.  A partition is a run of `PB` logical blocks; its four warps
// take its blocks round-robin, each warp with its own TMA pipeline of NST
// stages (one physical block's K tile and V tile per stage, 128-byte swizzled
// so the shared-memory reads below are bank-conflict free) and its own online
// softmax state.  The warps' states merge through shared memory at the end;
// the CTA then writes the output row (one partition) or a partial
// (running max, running sum, normalised output) for the merge kernel.
#pragma once

#include "ptx.cuh"

namespace pkv {

struct DecodeParams {
    void* out;
    const void* query;
    const int32_t* block_tables;
    const int32_t* context_lens;
    float* ws_max;    // [num_seqs, Hq, P]   (log2 domain)
    float* ws_sum;    // [num_seqs, Hq, P]
    float* ws_out;    // [num_seqs, Hq, P, D]
    float scale_log2; // scale * log2(e) (times the K pool's scale for FP8 pools)
    float out_scale;  // the V pool's scale for FP8 pools, else 1
    int num_seqs;
    int num_q_heads;
    int num_kv_heads;
    int max_blocks_per_seq;
    int64_t num_blocks;
    int partition_blocks;  // PB
    int num_partitions;    // P (grid extent)
};

template <typename T, int D, int B, int G, int NST, int NW>
struct DecodeCfg {
    static constexpr int WARPS = NW;
    static constexpr int THREADS = NW * 32;
    static constexpr int TB = Elem<T>::kBytes;
    static constexpr int PANEL = 128 / TB;              // elements per 128-byte swizzle row
    static constexpr int NP = D * TB / 128;             // panels per row
    static constexpr int TILE = B * D * TB;             // one block-head of K (or V)
    static constexpr int STAGE = 2 * TILE;
    static constexpr int E = 16 / TB;                   // elements per 16-byte chunk
    static constexpr int NCH = D / E;                   // chunks per row
    static constexpr int LPT = 32 / B;                  // lanes per token in Q.K
    static constexpr int CPL = NCH / LPT;               // chunks per lane in Q.K
    static constexpr int DPL = D / 32;                  // output dims per lane in P.V
    static constexpr int STAGES_BYTES = NW * NST * STAGE;
    static constexpr int Q_OFF = STAGES_BYTES;
    static constexpr int BT_OFF = Q_OFF + G * D * 4;
    static constexpr int RED_BYTES = NW * G * (D + 2) * 4;
    static_assert(TILE % 1024 == 0, "tiles must keep 1024-byte alignment for the 128-byte swizzle");
    static_assert(NCH % LPT == 0 && D % 32 == 0 && B <= 32, "unsupported decode shape");
    static_assert(RED_BYTES <= STAGES_BYTES, "merge scratch must fit in the stage buffers");
    static size_t smem_bytes(int pb) {
        return 1024 + BT_OFF + static_cast<size_t>(pb) * 4 + 16 + NW * NST * 8;
    }
};

// Number of logical blocks of a sequence the launch covers (clamped, flagged).
__device__ __forceinline__ int decode_seq_blocks(int ctx, int block_size, int max_blocks, int covered_blocks,
                                                 bool report) {
    int n = ctx;
    bool bad = false;
    if (n < 0) n = 0, bad = true;
    int nb = (n + block_size - 1) / block_size;
    if (nb > max_blocks) nb = max_blocks, bad = true;
    if (nb > covered_blocks) nb = covered_blocks, bad = true;
    if (bad && report) flag_error(PKV_DEVERR_LENGTH);
    return nb;
}

// Combine the NW warps' (max, sum, output) states of one CTA, left in
// shared memory as red_m[w][h], red_l[w][h], red_o[w][h][D], and write the
// output row (single partition) or the partition's partial to the workspace.
template <typename T, int D, int G, int NW>
__device__ __forceinline__ void decode_finish(const DecodeParams& p, const float* red_m, int s, int g, int part,
                                              bool direct) {
    const float* red_l = red_m + NW * G;
    const float* red_o = red_l + NW * G;
    const int64_t row0 = static_cast<int64_t>(s) * p.num_q_heads + static_cast<int64_t>(g) * G;
    for (int i = threadIdx.x; i < G * D; i += NW * 32) {
        const int h = i / D, d = i - h * D;
        float mx = -INFINITY;
#pragma unroll
        for (int w = 0; w < NW; ++w) mx = fmaxf(mx, red_m[w * G + h]);
        float sum = 0.f, o = 0.f;
        if (mx != -INFINITY) {
#pragma unroll
            for (int w = 0; w < NW; ++w) {
                const float mw = red_m[w * G + h];
                if (mw != -INFINITY) {
                    const float f = exp2f(mw - mx);
                    sum += red_l[w * G + h] * f;
                    o += red_o[(w * G + h) * D + d] * f;
                }
            }
        }
        const float val = mx != -INFINITY ? o / sum * p.out_scale : 0.f;
        if (direct) {
            reinterpret_cast<T*>(p.out)[(row0 + h) * D + d] = Elem<T>::from_f(val);
        } else {
            const int64_t pi = (row0 + h) * p.num_partitions + part;
            p.ws_out[pi * D + d] = val;
            if (d == 0) {
                p.ws_max[pi] = mx;
                p.ws_sum[pi] = sum;
            }
        }
    }
}

template <typename T, int D, int B, int G, int NST, int NW>
__global__ void __launch_bounds__(NW * 32) paged_decode_kernel(const DecodeParams p,
                                                                      const __grid_constant__ CUtensorMap tm_k,
                                                                      const __grid_constant__ CUtensorMap tm_v) {
    using C = DecodeCfg<T, D, B, G, NST, NW>;
    constexpr int kDecodeWarps = NW;
    constexpr int kDecodeThreads = NW * 32;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align_1024(smem_raw);

    const int per_seq = p.num_partitions * p.num_kv_heads;
    const int s = blockIdx.x / per_seq;
    const int rem = blockIdx.x - s * per_seq;
    const int part = rem / p.num_kv_heads;
    const int g = rem - part * p.num_kv_heads;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    const int ctx_raw = p.context_lens[s];
    const int nblk = decode_seq_blocks(ctx_raw, B, p.max_blocks_per_seq, p.num_partitions * p.partition_blocks,
                                       threadIdx.x == 0 && part == 0 && g == 0);
    const int ctx = min(max(ctx_raw, 0), nblk * B);
    const int nparts = nblk > 0 ? (nblk + p.partition_blocks - 1) / p.partition_blocks : 1;
    if (part >= nparts) return;
    const int b0 = part * p.partition_blocks;
    const int nb = max(0, min(nblk - b0, p.partition_blocks));
    const bool direct = nparts == 1;

    float* q_s = reinterpret_cast<float*>(smem + C::Q_OFF);
    int* bt_s = reinterpret_cast<int*>(smem + C::BT_OFF);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + ((C::BT_OFF + p.partition_blocks * 4 + 15) & ~15));

    // Stage this group's query heads (fp32, pre-scaled into the log2 domain).
    const T* qg = reinterpret_cast<const T*>(p.query) +
                  (static_cast<int64_t>(s) * p.num_q_heads + static_cast<int64_t>(g) * G) * D;
    for (int i = threadIdx.x; i < G * D; i += kDecodeThreads) q_s[i] = Elem<T>::to_f(qg[i]) * p.scale_log2;
    // Stage this partition's physical block ids; out-of-range ids become -1.
    const int32_t* bt_row = p.block_tables + static_cast<int64_t>(s) * p.max_blocks_per_seq + b0;
    for (int i = threadIdx.x; i < nb; i += kDecodeThreads) {
        int id = bt_row[i];
        if (id < 0 || id >= p.num_blocks) {
            flag_error(PKV_DEVERR_BLOCK_ID);
            id = -1;
        }
        bt_s[i] = id;
    }
    if (lane == 0) {
#pragma unroll
        for (int st = 0; st < NST; ++st) mbar_init(&bars[warp * NST + st], 1);
        fence_mbar_init();
    }
    __syncthreads();

    // ---- per-warp streaming over blocks warp, warp + 4, ...
    const int nw = nb > warp ? (nb - warp + kDecodeWarps - 1) / kDecodeWarps : 0;
    uint8_t* wstage = smem + warp * NST * C::STAGE;
    uint64_t* wbar = bars + warp * NST;
    const uint64_t policy = l2_policy_evict_first();

    auto issue = [&](int k) {  // lane 0 only
        const int st = k % NST;
        const int id = bt_s[warp + k * kDecodeWarps];
        const int coord = id >= 0 ? id : static_cast<int>(p.num_blocks);  // out of range: zero fill
        uint8_t* kd = wstage + st * C::STAGE;
        uint8_t* vd = kd + C::TILE;
        mbar_arrive_expect_tx(&wbar[st], C::STAGE);
#pragma unroll
        for (int pn = 0; pn < C::NP; ++pn) {
            tma_load_4d_hint(kd + pn * B * 128, &tm_k, pn * C::PANEL, g, 0, coord, &wbar[st], policy);
            tma_load_4d_hint(vd + pn * B * 128, &tm_v, pn * C::PANEL, g, 0, coord, &wbar[st], policy);
        }
    };

    // Everything above reads only the query, the tables and the lengths; the
    // pools may still be in the writes of a grid this one depends on (the
    // append of a decode step), so their loads start after it completes.
    griddep_wait();
    if (lane == 0) {
        for (int k = 0; k < NST && k < nw; ++k) issue(k);
    }
    __syncwarp();

    float m[G], l[G], acc[G][C::DPL];
#pragma unroll
    for (int h = 0; h < G; ++h) {
        m[h] = -INFINITY;
        l[h] = 0.f;
#pragma unroll
        for (int j = 0; j < C::DPL; ++j) acc[h][j] = 0.f;
    }

    const int t = lane % B;   // token of this lane in Q.K
    const int tp = lane / B;  // which part of the row
    const int pd0 = lane * C::DPL;  // first output dim of this lane in P.V
    const int pc = pd0 / C::E;
    const int pv_off = (pc / 8) * B * 128 + (pd0 % C::E) * C::TB;
    const int pv_cc = pc % 8;

    int k = 0;
    for (; k < nw; ++k) {
        const int st = k % NST;
        const bool ok = mbar_wait_main(&wbar[st], (k / NST) & 1);
        if (!__all_sync(0xffffffffu, ok)) break;
        const int lb = b0 + warp + k * kDecodeWarps;
        const int valid = min(B, ctx - lb * B);
        if (bt_s[warp + k * kDecodeWarps] >= 0) {
            const uint8_t* Ks = wstage + st * C::STAGE;
            const uint8_t* Vs = Ks + C::TILE;
            // ---- scores: lane (t, tp) covers chunks tp, tp + LPT, ... of token t
            float x[G];
#pragma unroll
            for (int h = 0; h < G; ++h) x[h] = 0.f;
#pragma unroll
            for (int i = 0; i < C::CPL; ++i) {
                const int c = tp + C::LPT * i;
                const uint4 raw =
                    *reinterpret_cast<const uint4*>(Ks + (c / 8) * B * 128 + t * 128 + (((c % 8) ^ (t & 7)) << 4));
                float kf[C::E];
                Elem<T>::unpack16(raw, kf);
#pragma unroll
                for (int h = 0; h < G; ++h) {
                    const float4* qp = reinterpret_cast<const float4*>(q_s + h * D + c * C::E);
#pragma unroll
                    for (int e = 0; e < C::E / 4; ++e) {
                        const float4 qq = qp[e];
                        x[h] = fmaf(qq.x, kf[4 * e + 0], x[h]);
                        x[h] = fmaf(qq.y, kf[4 * e + 1], x[h]);
                        x[h] = fmaf(qq.z, kf[4 * e + 2], x[h]);
                        x[h] = fmaf(qq.w, kf[4 * e + 3], x[h]);
                    }
                }
            }
#pragma unroll
            for (int off = B; off < 32; off <<= 1)
#pragma unroll
                for (int h = 0; h < G; ++h) x[h] += __shfl_xor_sync(0xffffffffu, x[h], off);
            const bool tv = t < valid;
            // ---- online softmax over this block's tokens
            float pr[G];
#pragma unroll
            for (int h = 0; h < G; ++h) {
                float bm = tv ? x[h] : -INFINITY;
#pragma unroll
                for (int off = 1; off < B; off <<= 1) bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, off));
                const float mn = fmaxf(m[h], bm);
                const float alpha = exp2f(m[h] - mn);
                pr[h] = tv ? exp2f(x[h] - mn) : 0.f;
                float ps = pr[h];
#pragma unroll
                for (int off = 1; off < B; off <<= 1) ps += __shfl_xor_sync(0xffffffffu, ps, off);
                l[h] = l[h] * alpha + ps;
                m[h] = mn;
#pragma unroll
                for (int j = 0; j < C::DPL; ++j) acc[h][j] *= alpha;
            }
            // ---- P.V: lane owns DPL consecutive output dims
#pragma unroll
            for (int tt = 0; tt < B; ++tt) {
                float pv[G];
#pragma unroll
                for (int h = 0; h < G; ++h) pv[h] = __shfl_sync(0xffffffffu, pr[h], tt);
                if (tt < valid) {
                    const uint8_t* vp = Vs + pv_off + tt * 128 + ((pv_cc ^ (tt & 7)) << 4);
                    float vf[C::DPL];
                    if constexpr (C::DPL * C::TB == 16) {
                        Elem<T>::unpack16(*reinterpret_cast<const uint4*>(vp), vf);
                    } else if constexpr (C::DPL * C::TB == 8) {
                        const uint2 r2 = *reinterpret_cast<const uint2*>(vp);
                        if constexpr (C::TB == 4) {
                            vf[0] = __uint_as_float(r2.x);
                            vf[1] = __uint_as_float(r2.y);
                        } else {
                            const float2 a = Elem<T>::pair(r2.x), b = Elem<T>::pair(r2.y);
                            vf[0] = a.x, vf[1] = a.y, vf[2] = b.x, vf[3] = b.y;
                        }
                    } else {  // 4 bytes: two 16-bit elements
                        const float2 a = Elem<T>::pair(*reinterpret_cast<const uint32_t*>(vp));
                        vf[0] = a.x, vf[1] = a.y;
                    }
#pragma unroll
                    for (int h = 0; h < G; ++h)
#pragma unroll
                        for (int j = 0; j < C::DPL; ++j) acc[h][j] = fmaf(pv[h], vf[j], acc[h][j]);
                }
            }
        }
        __syncwarp();
        if (lane == 0 && k + NST < nw) {
            fence_proxy_async();
            issue(k + NST);
        }
    }
    if (k < nw && lane == 0) {
        // A wait gave up: wait (bounded) for the copies still in flight before
        // the stage buffers are reused, then drop this warp's partial state.
        // a wait gave up: wait (bounded) for this warp's copies still in flight, stage k's included
        for (int kk = k; kk < min(nw, k + NST); ++kk) mbar_wait(&wbar[kk % NST], (kk / NST) & 1);
    }
    if (k < nw) {
#pragma unroll
        for (int h = 0; h < G; ++h) m[h] = -INFINITY, l[h] = 0.f;
    }

    // ---- merge the four warps' states
    __syncthreads();
    float* red_m = reinterpret_cast<float*>(smem);
    float* red_l = red_m + kDecodeWarps * G;
    float* red_o = red_l + kDecodeWarps * G;
    if (lane == 0) {
#pragma unroll
        for (int h = 0; h < G; ++h) {
            red_m[warp * G + h] = m[h];
            red_l[warp * G + h] = l[h];
        }
    }
#pragma unroll
    for (int h = 0; h < G; ++h)
#pragma unroll
        for (int j = 0; j < C::DPL; ++j) red_o[(warp * G + h) * D + pd0 + j] = acc[h][j];
    __syncthreads();

    decode_finish<T, D, G, NW>(p, red_m, s, g, part, direct);
}

// ---- log-sum-exp merge of the partitions: one warp per (sequence, q head).
struct MergeParams {
    void* out;
    const int32_t* context_lens;
    const float* ws_max;
    const float* ws_sum;
    const float* ws_out;
    int num_seqs;
    int num_q_heads;
    int block_size;
    int max_blocks_per_seq;
    int partition_blocks;
    int num_partitions;
};

template <typename T, int D>
__global__ void __launch_bounds__(128) paged_decode_merge_kernel(const MergeParams p) {
    const int wid = blockIdx.x * 4 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (wid >= p.num_seqs * p.num_q_heads) return;
    const int s = wid / p.num_q_heads;
    const int nblk = decode_seq_blocks(p.context_lens[s], p.block_size, p.max_blocks_per_seq,
                                       p.num_partitions * p.partition_blocks, false);
    const int nparts = nblk > 0 ? (nblk + p.partition_blocks - 1) / p.partition_blocks : 1;
    if (nparts <= 1) return;  // the decode kernel wrote this row itself
    griddep_wait();           // the partials are the writes of the decode grid
    const float* pm = p.ws_max + static_cast<int64_t>(wid) * p.num_partitions;
    const float* pl = p.ws_sum + static_cast<int64_t>(wid) * p.num_partitions;
    const float* po = p.ws_out + static_cast<int64_t>(wid) * p.num_partitions * D;

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
        if constexpr (DPL == 4) {
            const float4 v = *reinterpret_cast<const float4*>(src);
            o[0] = fmaf(w, v.x, o[0]), o[1] = fmaf(w, v.y, o[1]), o[2] = fmaf(w, v.z, o[2]),
            o[3] = fmaf(w, v.w, o[3]);
        } else {
#pragma unroll
            for (int j = 0; j < DPL; ++j) o[j] = fmaf(w, src[j], o[j]);
        }
    }
    const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
    T* dst = reinterpret_cast<T*>(p.out) + static_cast<int64_t>(wid) * D + lane * DPL;
#pragma unroll
    for (int j = 0; j < DPL; ++j) dst[j] = Elem<T>::from_f(o[j] * inv);
}

}  // namespace pkv
