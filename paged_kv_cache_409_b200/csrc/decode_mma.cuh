// decode_mma.cuh -- paged decode attention for fp16 / bf16 (G = 1, 2, 4 or 8
// query heads per KV head) with the two small products on warp-level
// tensor-core MMAs (mma.sync m16n8k16, fp32 accumulation).
//
// With G query heads per KV head the decode kernel does 4 * G flops per K/V
// byte; on CUDA cores that is more instruction issue than a B200 SM has at
// HBM speed for G >= 4, and even at G = 1 the MMA form leaves more issue
// slots to the memory pipeline (measured 6.6 vs 6.2 TB/s on a 64-sequence,
// 32-head batch).  The contraction per physical block is tiny (16
// tokens x 128 dims x G heads), far below the 64/128-row minimum of tcgen05,
// so it goes to mma.sync instead:
//   S^T [16 tokens x 8 heads]  = K_tile [16 x D] . Q^T [D x 8]      (A: ldmatrix of K)
//   O^T [16 dims x 8 heads]   += V^T [16 x 16 tokens] . P^T [16 x 8] (A: ldmatrix.trans of V)
// Heads beyond G are zero padding.  P^T comes from the S^T accumulator by an
// in-register 8x8 transpose (movmatrix).  For bf16 the weights go in as two
// bf16 terms (hi + lo) so that their rounding stays below the output
// tolerance.  Everything else (partitions, per-warp TMA pipelines, the
// cross-warp merge, the workspace partials) is the same as the CUDA-core
// decode kernel in decode.cuh.
#pragma once

#include "decode.cuh"

namespace pkv {

template <typename T, int D, int B, int G, int NST, int NW>
__global__ void __launch_bounds__(NW * 32) paged_decode_mma_kernel(const DecodeParams p,
                                                                          const __grid_constant__ CUtensorMap tm_k,
                                                                          const __grid_constant__ CUtensorMap tm_v) {
    using C = DecodeCfg<T, D, B, G, NST, NW>;
    constexpr int kDecodeWarps = NW;
    constexpr int kDecodeThreads = NW * 32;
    constexpr bool kBf16 = Elem<T>::kCuType == CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    constexpr int KS = D / 16;            // 16-dim steps of Q.K^T; 16-dim tiles of O^T
    constexpr int MT = (B + 15) / 16;     // 16-token tiles per block
    static_assert(sizeof(T) == 2 && G >= 1 && G <= 8, "tensor-core decode takes 16-bit inputs and 1..8 heads");
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

    const int nw = nb > warp ? (nb - warp + kDecodeWarps - 1) / kDecodeWarps : 0;
    uint8_t* wstage = smem + warp * NST * C::STAGE;
    uint64_t* wbar = bars + warp * NST;
    const uint64_t policy = l2_policy_evict_first();

    auto issue = [&](int k) {  // lane 0 only
        const int st = k % NST;
        const int id = bt_s[warp + k * kDecodeWarps];
        const int coord = id >= 0 ? id : static_cast<int>(p.num_blocks);
        uint8_t* kd = wstage + st * C::STAGE;
        uint8_t* vd = kd + C::TILE;
        mbar_arrive_expect_tx(&wbar[st], C::STAGE);
#pragma unroll
        for (int pn = 0; pn < C::NP; ++pn) {
            tma_load_4d_hint(kd + pn * B * 128, &tm_k, pn * C::PANEL, g, 0, coord, &wbar[st], policy);
            tma_load_4d_hint(vd + pn * B * 128, &tm_v, pn * C::PANEL, g, 0, coord, &wbar[st], policy);
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
    // Q^T fragments (B operand), loaded while the first stages are in flight:
    // this lane holds head lane/4, dims 2(lane%4)+{0,1} (+8) of every 16-dim step.
    uint32_t qf[KS][2];
    {
        const int hq = lane >> 2, kq = 2 * (lane & 3);
        const T* qrow = reinterpret_cast<const T*>(p.query) +
                        (static_cast<int64_t>(s) * p.num_q_heads + static_cast<int64_t>(g) * G + hq) * D;
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {
            qf[ks][0] = hq < G ? *reinterpret_cast<const uint32_t*>(qrow + 16 * ks + kq) : 0u;
            qf[ks][1] = hq < G ? *reinterpret_cast<const uint32_t*>(qrow + 16 * ks + 8 + kq) : 0u;
        }
    }

    // Columns of S^T held by this lane: heads hA = 2(lane%4) and hB = hA + 1.
    float mA = -INFINITY, mB = -INFINITY, lA = 0.f, lB = 0.f;
    float o[KS][4];  // O^T: [dim tile][c0: (d, hA), c1: (d, hB), c2: (d + 8, hA), c3: (d + 8, hB)], d = 16 t + lane/4
#pragma unroll
    for (int t = 0; t < KS; ++t) o[t][0] = o[t][1] = o[t][2] = o[t][3] = 0.f;

    // ldmatrix row addresses: lane provides row (lane % 8) of matrix (lane / 8).
    const int lr = lane & 7, lm = lane >> 3;

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
            // ---- S^T = K . Q^T
            float sc[MT][4];
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
                // two accumulator chains (even / odd 16-dim steps) halve the
                // dependent MMA chain
                float sc2[4] = {0.f, 0.f, 0.f, 0.f};
                sc[mt][0] = sc[mt][1] = sc[mt][2] = sc[mt][3] = 0.f;
#pragma unroll
                for (int ks = 0; ks < KS; ++ks) {
                    uint32_t a[4];
                    if constexpr (B >= 16) {
                        const int tok = 16 * mt + lr + 8 * (lm & 1);
                        const int ch = 2 * ks + (lm >> 1);
                        ldsm_x4(a, Ks + (ch / 8) * B * 128 + tok * 128 + (((ch % 8) ^ (tok & 7)) << 4));
                    } else {
                        const int tok = lr;
                        const int ch = 2 * ks + (lm & 1);
                        ldsm_x2(a[0], a[2], Ks + (ch / 8) * B * 128 + tok * 128 + (((ch % 8) ^ (tok & 7)) << 4));
                        a[1] = a[3] = 0u;
                    }
                    if (ks & 1)
                        mma_16816<kBf16>(sc2, a, qf[ks][0], qf[ks][1]);
                    else
                        mma_16816<kBf16>(sc[mt], a, qf[ks][0], qf[ks][1]);
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
            // 2^8; the weights exp2(s - m) then stay below 256 (bf16 / f16 P).
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
                    o[t][2] *= alA;
                    o[t][1] *= alB;
                    o[t][3] *= alB;
                }
            }
            // ---- O^T += V^T . P^T
#pragma unroll
            for (int kt = 0; kt < MT; ++kt) {
                // P^T fragments (B operand): tokens 2(lane%4)+{0,1} (+8) of head lane/4
                const uint32_t h01 = Elem<T>::pack(sc[kt][0], sc[kt][1]);
                const uint32_t h23 = Elem<T>::pack(sc[kt][2], sc[kt][3]);
                const uint32_t bh0 = movmatrix_trans(h01), bh1 = movmatrix_trans(h23);
                uint32_t bl0 = 0, bl1 = 0;
                if constexpr (kBf16) {
                    const float2 f01 = Elem<T>::pair(h01), f23 = Elem<T>::pair(h23);
                    bl0 = movmatrix_trans(Elem<T>::pack(sc[kt][0] - f01.x, sc[kt][1] - f01.y));
                    bl1 = movmatrix_trans(Elem<T>::pack(sc[kt][2] - f23.x, sc[kt][3] - f23.y));
                }
                // tokens of this lane's V^T fragment halves, for masking a partial block
                const int t0 = 16 * kt + 2 * (lane & 3);
                const bool partial = valid < 16 * kt + 16;
#pragma unroll
                for (int t = 0; t < KS; ++t) {
                    uint32_t a[4];
                    if constexpr (B >= 16) {
                        const int tok = 16 * kt + lr + 8 * (lm >> 1);
                        const int ch = 2 * t + (lm & 1);
                        ldsm_x4_trans(a, Vs + (ch / 8) * B * 128 + tok * 128 + (((ch % 8) ^ (tok & 7)) << 4));
                    } else {
                        const int tok = lr;
                        const int ch = 2 * t + (lm & 1);
                        ldsm_x2_trans(a[0], a[1], Vs + (ch / 8) * B * 128 + tok * 128 + (((ch % 8) ^ (tok & 7)) << 4));
                        a[2] = a[3] = 0u;
                    }
                    if (partial) {  // rows past the context may hold anything: 0 * NaN must not reach O
                        const uint32_t m0 = (t0 < valid ? 0x0000FFFFu : 0u) | (t0 + 1 < valid ? 0xFFFF0000u : 0u);
                        const uint32_t m1 =
                            (t0 + 8 < valid ? 0x0000FFFFu : 0u) | (t0 + 9 < valid ? 0xFFFF0000u : 0u);
                        a[0] &= m0;
                        a[1] &= m0;
                        a[2] &= m1;
                        a[3] &= m1;
                    }
                    mma_16816<kBf16>(o[t], a, bh0, bh1);
                    if constexpr (kBf16) mma_16816<kBf16>(o[t], a, bl0, bl1);
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
    float* red_l = red_m + kDecodeWarps * G;
    float* red_o = red_l + kDecodeWarps * G;
    const int hA = 2 * (lane & 3), hB = hA + 1;
    if (lane < 4) {
        if (hA < G) red_m[warp * G + hA] = mA, red_l[warp * G + hA] = lA;
        if (hB < G) red_m[warp * G + hB] = mB, red_l[warp * G + hB] = lB;
    }
#pragma unroll
    for (int t = 0; t < KS; ++t) {
        const int d = 16 * t + (lane >> 2);
        if (hA < G) {
            red_o[(warp * G + hA) * D + d] = o[t][0];
            red_o[(warp * G + hA) * D + d + 8] = o[t][2];
        }
        if (hB < G) {
            red_o[(warp * G + hB) * D + d] = o[t][1];
            red_o[(warp * G + hB) * D + d + 8] = o[t][3];
        }
    }
    __syncthreads();
    decode_finish<T, D, G, NW>(p, red_m, s, g, part, direct);
}

}  // namespace pkv
