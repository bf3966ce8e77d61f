// decode_fp8.cuh -- paged decode attention over FP8 (E4M3) K/V pools, head
// dim 128, query and output in fp16 or bf16, 1 to 8 query heads per KV head.
//
// An FP8 pool halves the bytes decode streams from HBM, so at HBM speed each
// SM has twice as many K/V elements per second to turn into products as with
// 16-bit pools.  Both products therefore run on warp MMAs (mma.sync m16n8k16,
// f16 inputs, fp32 accumulation) for every grouping, one head included:
//   S^T [16 tokens x 8 heads] = K_tile . Q^T,   O^T [16 dims x 8 heads] += V^T . P^T.
// Every E4M3 value is exactly an f16 value, so K and V are widened with
// cvt.f16x2.e4m3x2 straight out of ldmatrix fragments:
//   * K: ldmatrix of the FP8 tile read as 16-bit pairs gives a lane four
//     consecutive dims (4c .. 4c+3) of one token.  The MMA contracts over any
//     fixed order of the dims, so those four become the lane's k slots
//     (2c, 2c+1, 2c+8, 2c+9) and the query fragment is loaded in the same
//     order.
//   * V: ldmatrix.trans of the same pairs gives a lane two tokens x two
//     adjacent dims; a byte permute regroups them per dim, and the two dims
//     become rows g and g + 8 of the lane's A fragment (row g = dim 2g, row
//     g + 8 = dim 2g + 1 of the 16-dim chunk) -- the output rows come back in
//     that order.
// The query is rounded to f16 once (a bf16 query keeps its 8 significant bits
// unless |q| < 2^-14; |q| must stay below 65504), the weights P go in as f16
// (11 significant bits, one MMA term).  The pools' scales fold into the
// score scale (k_scale) and the final normalisation (v_scale).  Partitions,
// per-warp TMA pipelines and the CTA merge are those of decode.cuh.
#pragma once

#include "decode.cuh"

namespace pkv {

// U consecutive blocks of a sequence form one unit (one stage, one softmax
// step): at block 16 with 4 or 8 heads per KV head, 32-token units give every
// step two independent 16-token S tiles and halve the per-block reductions,
// shuffles and waits.
template <int B, int G, int NST, int NW, int U>
struct DecodeFp8Cfg {
    static constexpr int D = 128;
    static constexpr int TILE = B * U * D;   // one unit-head of K (or V): B * U rows of 128 bytes
    static constexpr int STAGE = 2 * TILE;
    static constexpr int STAGES_BYTES = NW * NST * STAGE;
    static constexpr int RED_BYTES = NW * G * (D + 2) * 4;  // the merge reuses the stage buffers
    static constexpr int BT_OFF = STAGES_BYTES > RED_BYTES ? STAGES_BYTES : RED_BYTES;
    static_assert(TILE % 1024 == 0, "tiles must keep 1024-byte alignment for the 128-byte swizzle");
    static size_t smem_bytes(int pb) { return 1024 + BT_OFF + static_cast<size_t>(pb) * 4 + 16 + NW * NST * 8; }
};

// Resident CTAs per SM the register allocation must allow (launch bounds).
#ifndef PKV_FP8_MIN_CTAS
#define PKV_FP8_MIN_CTAS 1
#endif

template <typename T, int B, int G, int NST, int NW, int U>
__global__ void __launch_bounds__(NW * 32, PKV_FP8_MIN_CTAS) paged_decode_fp8_kernel(const DecodeParams p,
                                                                   const __grid_constant__ CUtensorMap tm_k,
                                                                   const __grid_constant__ CUtensorMap tm_v) {
    using C = DecodeFp8Cfg<B, G, NST, NW, U>;
    constexpr int D = C::D;
    constexpr int kThreads = NW * 32;
    constexpr int KS = D / 16;          // 16-dim chunks
    constexpr int BU = B * U;           // tokens per unit
    constexpr int MT = (BU + 15) / 16;  // 16-token tiles per unit
    static_assert(sizeof(T) == 2 && G >= 1 && G <= 8, "FP8 decode takes a 16-bit query and 1..8 heads");
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

    int* bt_s = reinterpret_cast<int*>(smem + C::BT_OFF);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + ((C::BT_OFF + p.partition_blocks * 4 + 15) & ~15));
    const int32_t* bt_row = p.block_tables + static_cast<int64_t>(s) * p.max_blocks_per_seq + b0;
    for (int i = threadIdx.x; i < nb; i += kThreads) {
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

    const int nu = (nb + U - 1) / U;  // units of the partition
    const int nw = nu > warp ? (nu - warp + NW - 1) / NW : 0;
    uint8_t* wstage = smem + warp * NST * C::STAGE;
    uint64_t* wbar = bars + warp * NST;
    const uint64_t policy = l2_policy_evict_first();

    auto issue = [&](int k) {  // lane 0 only
        const int st = k % NST;
        uint8_t* kd = wstage + st * C::STAGE;
        mbar_arrive_expect_tx(&wbar[st], C::STAGE);
#pragma unroll
        for (int i = 0; i < U; ++i) {
            const int bi = (warp + k * NW) * U + i;
            const int id = bi < nb ? bt_s[bi] : -1;
            const int coord = id >= 0 ? id : static_cast<int>(p.num_blocks);  // out of range: zero fill
            tma_load_4d_hint(kd + i * B * 128, &tm_k, 0, g, 0, coord, &wbar[st], policy);
            tma_load_4d_hint(kd + C::TILE + i * B * 128, &tm_v, 0, g, 0, coord, &wbar[st], policy);
        }
    };
    // Everything above reads only the tables and the lengths; the
    // pools may still be in the writes of a grid this one depends on (the
    // append of a decode step), so their loads start after it completes.
    griddep_wait();
    if (lane == 0) {
        for (int k = 0; k < NST && k < nw; ++k) issue(k);
    }
    __syncwarp();
    // Q^T fragments (B operand, f16), loaded while the first stages are in
    // flight: head lane/4, dims 16 ks + 4 (lane%4) + {0,1} | {2,3}.
    uint32_t qf[KS][2];
    {
        const int hq = lane >> 2, k4 = 4 * (lane & 3);
        const T* qrow = reinterpret_cast<const T*>(p.query) +
                        (static_cast<int64_t>(s) * p.num_q_heads + static_cast<int64_t>(g) * G + hq) * D;
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {
            if (hq < G) {
                const uint2 raw = *reinterpret_cast<const uint2*>(qrow + 16 * ks + k4);
                const float2 a = Elem<T>::pair(raw.x), b = Elem<T>::pair(raw.y);
                qf[ks][0] = pack_half2(a.x, a.y);
                qf[ks][1] = pack_half2(b.x, b.y);
            } else {
                qf[ks][0] = qf[ks][1] = 0u;
            }
        }
    }

    float mA = -INFINITY, mB = -INFINITY, lA = 0.f, lB = 0.f;
    // O^T: [chunk t][c0: (dim 16t + 2(lane/4), hA), c1: (same dim, hB), c2: (dim + 1, hA), c3: (dim + 1, hB)]
    float o[KS][4];
#pragma unroll
    for (int t = 0; t < KS; ++t) o[t][0] = o[t][1] = o[t][2] = o[t][3] = 0.f;

    const int lr = lane & 7, lm = lane >> 3;

    int k = 0;
    for (; k < nw; ++k) {
        const int st = k % NST;
        const bool ok = mbar_wait_main(&wbar[st], (k / NST) & 1);
        if (!__all_sync(0xffffffffu, ok)) break;
        const int u0 = (warp + k * NW) * U;  // the unit's first block in the partition
        const int lb = b0 + u0;
        // the unit's keys end at the partition's end or at a bad block id
        // (flagged when the table was staged); the rest was loaded as zeros
        int valid = min(BU, ctx - lb * B);
#pragma unroll
        for (int i = 1; i < U; ++i)
            if (u0 + i >= nb || bt_s[u0 + i] < 0) valid = min(valid, i * B);
        if (bt_s[u0] >= 0) {
            const uint8_t* Ks = wstage + st * C::STAGE;
            const uint8_t* Vs = Ks + C::TILE;
            // ---- S^T = K . Q^T
            float sc[MT][4];
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
                // two accumulator chains (the h = 0 and h = 1 halves of each
                // 32-dim step) halve the dependent MMA chain
                float sc2[4] = {0.f, 0.f, 0.f, 0.f};
                sc[mt][0] = sc[mt][1] = sc[mt][2] = sc[mt][3] = 0.f;
#pragma unroll
                for (int kp = 0; kp < KS / 2; ++kp) {
                    // r[0]: token g, chunk 2kp; r[1]: token g + 8, chunk 2kp; r[2], r[3]: chunk 2kp + 1
                    uint32_t r[4];
                    if constexpr (BU >= 16) {
                        const int tok = 16 * mt + lr + 8 * (lm & 1);
                        const int ch = 2 * kp + (lm >> 1);
                        ldsm_x4(r, Ks + tok * 128 + ((ch ^ (tok & 7)) << 4));
                    } else {
                        const int tok = lr;
                        const int ch = 2 * kp + (lm & 1);
                        ldsm_x2(r[0], r[2], Ks + tok * 128 + ((ch ^ (tok & 7)) << 4));
                        r[1] = r[3] = 0u;
                    }
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const uint32_t top = r[2 * h], bot = r[2 * h + 1];
                        const uint32_t a[4] = {f16x2_from_e4m3x2(static_cast<uint16_t>(top)),
                                               f16x2_from_e4m3x2(static_cast<uint16_t>(bot)),
                                               f16x2_from_e4m3x2(static_cast<uint16_t>(top >> 16)),
                                               f16x2_from_e4m3x2(static_cast<uint16_t>(bot >> 16))};
                        if (h == 0)
                            mma_16816<false>(sc[mt], a, qf[2 * kp + h][0], qf[2 * kp + h][1]);
                        else
                            mma_16816<false>(sc2, a, qf[2 * kp + h][0], qf[2 * kp + h][1]);
                    }
                }
#pragma unroll
                for (int e = 0; e < 4; ++e) sc[mt][e] += sc2[e];
            }
            // ---- online softmax per head column (log2 domain)
            float bmA = -INFINITY, bmB = -INFINITY;
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int tok = 16 * mt + (lane >> 2) + (j >= 2 ? 8 : 0);
                    sc[mt][j] = tok < valid ? sc[mt][j] * p.scale_log2 : -INFINITY;
                }
                bmA = fmaxf(bmA, fmaxf(sc[mt][0], sc[mt][2]));
                bmB = fmaxf(bmB, fmaxf(sc[mt][1], sc[mt][3]));
            }
#pragma unroll
            for (int off = 4; off < 32; off <<= 1) {
                bmA = fmaxf(bmA, __shfl_xor_sync(0xffffffffu, bmA, off));
                bmB = fmaxf(bmB, __shfl_xor_sync(0xffffffffu, bmB, off));
            }
            // Lazy rescaling: the exponent base (mA, mB) moves, and O and the
            // sums are rescaled, only when a block's max exceeds it by more than
            // 2^8; the weights exp2(s - m) then stay below 256, inside f16.
            const bool rsA = bmA > mA + 8.f || (mA == -INFINITY && bmA != -INFINITY);
            const bool rsB = bmB > mB + 8.f || (mB == -INFINITY && bmB != -INFINITY);
            float alA = 1.f, alB = 1.f;
            if (rsA) alA = ex2_approx(mA - bmA), mA = bmA;  // 0 when mA was -inf
            if (rsB) alB = ex2_approx(mB - bmB), mB = bmB;
            const float eA = mA == -INFINITY ? 0.f : mA, eB = mB == -INFINITY ? 0.f : mB;
            float sA = 0.f, sB = 0.f;
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
                sc[mt][0] = ex2_approx(sc[mt][0] - eA);
                sc[mt][1] = ex2_approx(sc[mt][1] - eB);
                sc[mt][2] = ex2_approx(sc[mt][2] - eA);
                sc[mt][3] = ex2_approx(sc[mt][3] - eB);
                sA += sc[mt][0] + sc[mt][2];
                sB += sc[mt][1] + sc[mt][3];
            }
#pragma unroll
            for (int off = 4; off < 32; off <<= 1) {
                sA += __shfl_xor_sync(0xffffffffu, sA, off);
                sB += __shfl_xor_sync(0xffffffffu, sB, off);
            }
            lA = lA * alA + sA;
            lB = lB * alB + sB;
            if (__any_sync(0xffffffffu, rsA || rsB)) {
#pragma unroll
                for (int t = 0; t < KS; ++t) {
                    o[t][0] *= alA;
                    o[t][1] *= alB;
                    o[t][2] *= alA;
                    o[t][3] *= alB;
                }
            }
            // ---- O^T += V^T . P^T
#pragma unroll
            for (int kt = 0; kt < MT; ++kt) {
                const uint32_t bh0 = movmatrix_trans(pack_half2(sc[kt][0], sc[kt][1]));
                const uint32_t bh1 = movmatrix_trans(pack_half2(sc[kt][2], sc[kt][3]));
                const int t0 = 16 * kt + 2 * (lane & 3);
                const bool partial = valid < 16 * kt + 16;
                const uint32_t m0 = (t0 < valid ? 0x0000FFFFu : 0u) | (t0 + 1 < valid ? 0xFFFF0000u : 0u);
                const uint32_t m1 = (t0 + 8 < valid ? 0x0000FFFFu : 0u) | (t0 + 9 < valid ? 0xFFFF0000u : 0u);
#pragma unroll
                for (int jp = 0; jp < KS / 2; ++jp) {
                    // r[0]: tokens 2c, 2c+1 x dims 2g, 2g+1 of chunk 2jp; r[1]: tokens + 8; r[2], r[3]: chunk 2jp + 1
                    uint32_t r[4];
                    if constexpr (BU >= 16) {
                        const int tok = 16 * kt + lr + 8 * (lm & 1);
                        const int ch = 2 * jp + (lm >> 1);
                        ldsm_x4_trans(r, Vs + tok * 128 + ((ch ^ (tok & 7)) << 4));
                    } else {
                        const int tok = lr;
                        const int ch = 2 * jp + (lm & 1);
                        ldsm_x2_trans(r[0], r[2], Vs + tok * 128 + ((ch ^ (tok & 7)) << 4));
                        r[1] = r[3] = 0u;
                    }
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        // bytes (tok 2c, dim 2g) (tok 2c, dim 2g+1) (tok 2c+1, dim 2g) (tok 2c+1, dim 2g+1)
                        // -> dim 2g: (tok 2c, tok 2c+1) in the low half, dim 2g+1 in the high half
                        const uint32_t lo = __byte_perm(r[2 * h], 0u, 0x3120);
                        const uint32_t hi = __byte_perm(r[2 * h + 1], 0u, 0x3120);
                        uint32_t a[4] = {f16x2_from_e4m3x2(static_cast<uint16_t>(lo)),
                                         f16x2_from_e4m3x2(static_cast<uint16_t>(lo >> 16)),
                                         f16x2_from_e4m3x2(static_cast<uint16_t>(hi)),
                                         f16x2_from_e4m3x2(static_cast<uint16_t>(hi >> 16))};
                        if (partial) {  // rows past the context may hold anything: 0 * NaN must not reach O
                            a[0] &= m0;
                            a[1] &= m0;
                            a[2] &= m1;
                            a[3] &= m1;
                        }
                        mma_16816<false>(o[2 * jp + h], a, bh0, bh1);
                    }
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
        // a wait gave up: wait (bounded) for this warp's copies still in flight, stage k's included
        for (int kk = k; kk < min(nw, k + NST); ++kk) mbar_wait(&wbar[kk % NST], (kk / NST) & 1);
    }
    if (k < nw) mA = mB = -INFINITY, lA = lB = 0.f;

    // ---- hand this warp's state to the CTA merge
    __syncthreads();
    float* red_m = reinterpret_cast<float*>(smem);
    float* red_l = red_m + NW * G;
    float* red_o = red_l + NW * G;
    const int hA = 2 * (lane & 3), hB = hA + 1;
    if (lane < 4) {
        if (hA < G) red_m[warp * G + hA] = mA, red_l[warp * G + hA] = lA;
        if (hB < G) red_m[warp * G + hB] = mB, red_l[warp * G + hB] = lB;
    }
#pragma unroll
    for (int t = 0; t < KS; ++t) {
        const int d = 16 * t + 2 * (lane >> 2);
        if (hA < G) {
            red_o[(warp * G + hA) * D + d] = o[t][0];
            red_o[(warp * G + hA) * D + d + 1] = o[t][2];
        }
        if (hB < G) {
            red_o[(warp * G + hB) * D + d] = o[t][1];
            red_o[(warp * G + hB) * D + d + 1] = o[t][3];
        }
    }
    __syncthreads();
    decode_finish<T, D, G, NW>(p, red_m, s, g, part, direct);
}

}  // namespace pkv
