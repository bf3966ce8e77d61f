/*
 * pagedkv_oracle.c -- plain, slow, double-precision CPU oracle for the paged
 * KV-cache hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path (the CUDA library
 * and its Python binding) may call, link or load this file; only the tests,
 * the smoke check and the benchmark's CPU-baseline leg do.  It shares no code,
 * header, table or constant with the CUDA library.
 *
 * Sources (all from the vLLM / PagedAttention pages):
 *  - "vLLM 与 PagedAttention" (inference.mavenzero.com/case-studies/vllm),
 *    section 二 "PagedAttention 的解法": the KV cache is cut into fixed-size
 *    blocks (16 tokens by default) and a per-request block table maps logical
 *    blocks to physical blocks scattered over one pool; blocks are taken on
 *    demand; requests with a common prefix point at the same physical blocks
 *    and copy on write.
 *  - same page, section 二 "注意力计算改造": K/V are loaded block by block
 *    instead of from one contiguous buffer, each block's attention is computed
 *    and the results accumulated; the kernel sketch there fixes the cache
 *    layout [num_blocks, block_size, num_heads, d_head] for both K and V and
 *    an int block_table of max_num_blocks_per_seq entries.
 *  - "指南" (illegalscreed.cn .../vllm/guide-line), "KV Cache 是什么": each
 *    generated token attends to all previous tokens' cached K and V.
 *  - same page, "Copy-on-Write" and "Chunked Prefill": shared blocks are
 *    copied only when a request diverges; long prompts are prefilled in chunks
 *    scheduled together with decode steps.
 *
 * The pages never write the attention formula.  Plainest reading (stated in
 * the design notes): standard scaled dot-product attention,
 *     out = sum_j softmax_j(scale * q . K_j) V_j,
 * over all cached positions j < context_len for decode, and over the causal
 * key set j <= c0 + i for query row i of a prefill chunk with c0 prior tokens.
 * The oracle gathers each sequence's blocks through its block table into a
 * contiguous K/V in double precision and evaluates that definition directly
 * (max subtraction only guards exp() against overflow; it does not change the
 * mathematical value).
 *
 * Element types: 0 = fp32, 1 = fp16 (IEEE binary16), 2 = bf16, 3 = FP8 E4M3
 * (cache pools only).  Every stored element is converted exactly to double
 * before any arithmetic.
 *
 * FP8 KV cache.  Both pages list FP8 (E4M3) among vLLM's quantisation modes
 * (case-study page, section 五 "量化支持", table row "FP8 (E4M3)"; guide page,
 * "量化": 8 bits, half the memory of FP16, close to lossless, native on Hopper)
 * but only for weights and activations and without a scaling rule.  Reading
 * used here for the cache: one scale per pool (k_scale, v_scale); a stored
 * code is the E4M3 value nearest to x / scale (ties to even, magnitudes above
 * the largest finite value 448 clamped to 448, NaN kept NaN); the value a
 * code stands for is scale * e4m3(code).  E4M3 itself is the OCP 8-bit
 * floating-point format: 1 sign bit, 4 exponent bits with bias 7, 3 mantissa
 * bits, subnormals at exponent field 0, no infinities, and the single NaN
 * pattern S.1111.111 per sign.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

enum { ORC_F32 = 0, ORC_F16 = 1, ORC_BF16 = 2, ORC_E4M3 = 3 };

/* Host threads the attention functions may use: n > 0 sets the number, any
 * n returns the number now in force (1 in a build without OpenMP). */
int oracle_num_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
    return omp_get_max_threads();
#else
    (void)n;
    return 1;
#endif
}

static int elem_bytes(int dtype) {
    switch (dtype) {
        case ORC_F32: return 4;
        case ORC_F16: return 2;
        case ORC_BF16: return 2;
        case ORC_E4M3: return 1;
        default: return 0;
    }
}

/* E4M3 code -> double, by the format's definition (exact). */
static double e4m3_bits_to_double(uint8_t c) {
    int sign = (c >> 7) & 1;
    int expo = (c >> 3) & 0xf;
    int mant = c & 0x7;
    double v;
    if (expo == 15 && mant == 7) {
        v = NAN;
    } else if (expo == 0) {
        v = ldexp((double)mant, -9);                /* 0.mant * 2^(1-7) = mant/8 * 2^-6 */
    } else {
        v = ldexp((double)(8 + mant), expo - 10);   /* 1.mant * 2^(e-7) */
    }
    return sign ? -v : v;
}

/* double -> E4M3 code: the nearest of the 127 non-negative finite values to
 * |x| (found by trying them all), ties to the even code (adjacent values have
 * adjacent codes, so this is ties-to-even-mantissa); magnitudes above 448 thus
 * go to 448, infinities included; the sign bit is the sign of x (so -0 and
 * negative values that round to zero give 0x80); NaN gives 0x7F. */
static uint8_t double_to_e4m3(double x) {
    if (isnan(x)) return 0x7F;
    uint8_t sign = signbit(x) ? 0x80 : 0x00;
    double a = fabs(x);
    int best = 0;
    double best_err = INFINITY;
    for (int c = 0; c <= 0x7E; ++c) {
        double err = fabs(e4m3_bits_to_double((uint8_t)c) - a);
        if (err < best_err || (err == best_err && (c & 1) == 0)) {
            best = c;
            best_err = err;
        }
    }
    return (uint8_t)(sign | best);
}

/* Exposed for the pins: codes of n doubles. */
int oracle_e4m3_encode(uint8_t* dst, const double* src, int64_t n) {
    if (n < 0) return -1;
    for (int64_t i = 0; i < n; ++i) dst[i] = double_to_e4m3(src[i]);
    return 0;
}

/* IEEE binary16 -> double, exact (every binary16 value is a double). */
static double half_bits_to_double(uint16_t h) {
    int sign = (h >> 15) & 1;
    int expo = (h >> 10) & 0x1f;
    int mant = h & 0x3ff;
    double v;
    if (expo == 0) {
        v = ldexp((double)mant, -24);                 /* zero or subnormal */
    } else if (expo == 31) {
        v = mant ? NAN : INFINITY;
    } else {
        v = ldexp((double)(1024 + mant), expo - 25);  /* 1.mant * 2^(e-15) */
    }
    return sign ? -v : v;
}

/* bfloat16 is the top half of an IEEE binary32. */
static double bf16_bits_to_double(uint16_t h) {
    uint32_t u = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

static double load_elem(const void* base, int64_t idx, int dtype) {
    if (dtype == ORC_F32) {
        float f;
        memcpy(&f, (const char*)base + idx * 4, 4);
        return (double)f;
    }
    if (dtype == ORC_E4M3) return e4m3_bits_to_double(((const uint8_t*)base)[idx]);
    uint16_t h;
    memcpy(&h, (const char*)base + idx * 2, 2);
    return dtype == ORC_F16 ? half_bits_to_double(h) : bf16_bits_to_double(h);
}

/* Exposed so tests can pin the element decoding against numpy / torch. */
int oracle_to_double(double* dst, const void* src, int64_t n, int dtype) {
    if (!elem_bytes(dtype) || n < 0) return -1;
    for (int64_t i = 0; i < n; ++i) dst[i] = load_elem(src, i, dtype);
    return 0;
}

/* ---------------------------------------------------------------------------
 * Block arithmetic ("PagedAttention 的解法"; "PagedKVCache" sketch on the
 * 298.name page): a sequence of n tokens needs ceil(n / block_size) blocks;
 * token position pos lives in logical block pos / block_size at offset
 * pos % block_size, i.e. in physical slot
 *     block_table[pos / block_size] * block_size + pos % block_size.
 * ------------------------------------------------------------------------- */
int64_t oracle_blocks_needed(int64_t num_tokens, int block_size) {
    if (block_size <= 0 || num_tokens < 0) return -1;
    int64_t blocks = 0;
    int64_t covered = 0;
    while (covered < num_tokens) {   /* count blocks one by one: no ceil trick */
        covered += block_size;
        blocks += 1;
    }
    return blocks;
}

int64_t oracle_slot_for_position(const int32_t* block_table_row, int64_t pos, int block_size) {
    if (block_size <= 0 || pos < 0) return -1;
    int64_t logical_block = pos / block_size;
    int64_t offset = pos - logical_block * block_size;
    return (int64_t)block_table_row[logical_block] * block_size + offset;
}

/* ---------------------------------------------------------------------------
 * reshape_and_cache: write token t's K row (num_kv_heads x head_dim elements)
 * and V row into physical slot slot_mapping[t] of the pools laid out as
 * [num_blocks, block_size, num_kv_heads, head_dim].  A negative slot marks a
 * padding token and is skipped.  Element bits are copied verbatim.
 * Returns 0, or -1 when a slot lies beyond the pool.
 * ------------------------------------------------------------------------- */
int oracle_reshape_and_cache(const void* key, const void* value, void* key_cache, void* value_cache,
                             const int64_t* slot_mapping, int64_t num_tokens, int num_kv_heads,
                             int head_dim, int block_size, int64_t num_blocks, int dtype) {
    int eb = elem_bytes(dtype);
    if (!eb) return -1;
    int64_t row_elems = (int64_t)num_kv_heads * head_dim;
    for (int64_t t = 0; t < num_tokens; ++t) {
        int64_t slot = slot_mapping[t];
        if (slot < 0) continue;
        if (slot >= num_blocks * block_size) return -1;
        int64_t block = slot / block_size;
        int64_t offset = slot % block_size;
        for (int h = 0; h < num_kv_heads; ++h) {
            for (int d = 0; d < head_dim; ++d) {
                int64_t src = t * row_elems + (int64_t)h * head_dim + d;
                int64_t dst = ((block * block_size + offset) * num_kv_heads + h) * (int64_t)head_dim + d;
                memcpy((char*)key_cache + dst * eb, (const char*)key + src * eb, eb);
                memcpy((char*)value_cache + dst * eb, (const char*)value + src * eb, eb);
            }
        }
    }
    return 0;
}

/* ---------------------------------------------------------------------------
 * reshape_and_cache into FP8 pools: as above, but each element x of token t's
 * K (V) row is stored as the E4M3 code of x / k_scale (x / v_scale); the
 * quotient is formed in double.  key/value are in src_dtype (fp32/fp16/bf16),
 * the pools hold one byte per element.
 * ------------------------------------------------------------------------- */
int oracle_reshape_and_cache_fp8(const void* key, const void* value, uint8_t* key_cache, uint8_t* value_cache,
                                 const int64_t* slot_mapping, int64_t num_tokens, int num_kv_heads,
                                 int head_dim, int block_size, int64_t num_blocks, int src_dtype,
                                 double k_scale, double v_scale) {
    if (src_dtype == ORC_E4M3 || !elem_bytes(src_dtype) || !(k_scale > 0.0) || !(v_scale > 0.0)) return -1;
    int64_t row_elems = (int64_t)num_kv_heads * head_dim;
    for (int64_t t = 0; t < num_tokens; ++t) {
        int64_t slot = slot_mapping[t];
        if (slot < 0) continue;
        if (slot >= num_blocks * block_size) return -1;
        int64_t block = slot / block_size;
        int64_t offset = slot % block_size;
        for (int h = 0; h < num_kv_heads; ++h) {
            for (int d = 0; d < head_dim; ++d) {
                int64_t src = t * row_elems + (int64_t)h * head_dim + d;
                int64_t dst = ((block * block_size + offset) * num_kv_heads + h) * (int64_t)head_dim + d;
                key_cache[dst] = double_to_e4m3(load_elem(key, src, src_dtype) / k_scale);
                value_cache[dst] = double_to_e4m3(load_elem(value, src, src_dtype) / v_scale);
            }
        }
    }
    return 0;
}

/* ---------------------------------------------------------------------------
 * copy_blocks (copy-on-write of a shared block): for every pair (src, dst)
 * in order, and for every layer's K and V pool, copy the whole physical block
 * src (block_bytes bytes) over block dst.  Returns -1 on an id outside the
 * pool.
 * ------------------------------------------------------------------------- */
int oracle_copy_blocks(void* const* key_caches, void* const* value_caches, int num_layers,
                       const int64_t* src_dst_pairs, int64_t num_pairs, int64_t block_bytes,
                       int64_t num_blocks) {
    for (int64_t p = 0; p < num_pairs; ++p) {
        int64_t src = src_dst_pairs[2 * p];
        int64_t dst = src_dst_pairs[2 * p + 1];
        if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) return -1;
        for (int l = 0; l < num_layers; ++l) {
            memmove((char*)key_caches[l] + dst * block_bytes, (char*)key_caches[l] + src * block_bytes,
                    (size_t)block_bytes);
            memmove((char*)value_caches[l] + dst * block_bytes, (char*)value_caches[l] + src * block_bytes,
                    (size_t)block_bytes);
        }
    }
    return 0;
}

/* Gather positions [0, n) of one sequence's KV head g into contiguous
 * K[n][head_dim], V[n][head_dim] (double), following the block table; each
 * element is its stored value times the pool's scale (1 for 16/32-bit
 * pools, which is exact). */
static int gather_sequence(double* Kc, double* Vc, const void* key_cache, const void* value_cache,
                           int dtype, double k_scale, double v_scale, const int32_t* bt_row, int64_t n, int g,
                           int num_kv_heads, int head_dim, int block_size, int max_blocks_per_seq,
                           int64_t num_blocks) {
    for (int64_t j = 0; j < n; ++j) {
        int64_t logical_block = j / block_size;
        int64_t offset = j % block_size;
        if (logical_block >= max_blocks_per_seq) return -1;
        int64_t physical = bt_row[logical_block];
        if (physical < 0 || physical >= num_blocks) return -1;
        int64_t row = ((physical * block_size + offset) * num_kv_heads + g) * (int64_t)head_dim;
        for (int d = 0; d < head_dim; ++d) {
            Kc[j * head_dim + d] = k_scale * load_elem(key_cache, row + d, dtype);
            Vc[j * head_dim + d] = v_scale * load_elem(value_cache, row + d, dtype);
        }
    }
    return 0;
}

/* softmax(scale * q . K_j) V over keys j < n of contiguous Kc/Vc; writes
 * head_dim doubles to o.  n == 0 gives zeros (empty attention). */
static void attend(double* o, const double* q, const double* Kc, const double* Vc, int64_t n,
                   int head_dim, double scale, double* x) {
    for (int d = 0; d < head_dim; ++d) o[d] = 0.0;
    if (n <= 0) return;
    double m = -INFINITY;
    for (int64_t j = 0; j < n; ++j) {
        double dot = 0.0;
        for (int d = 0; d < head_dim; ++d) dot += q[d] * Kc[j * head_dim + d];
        x[j] = scale * dot;
        if (x[j] > m) m = x[j];
    }
    double denom = 0.0;
    for (int64_t j = 0; j < n; ++j) {
        x[j] = exp(x[j] - m);
        denom += x[j];
    }
    for (int64_t j = 0; j < n; ++j) {
        double w = x[j] / denom;
        for (int d = 0; d < head_dim; ++d) o[d] += w * Vc[j * head_dim + d];
    }
}

/* ---------------------------------------------------------------------------
 * Decode: one query token per sequence.  out[s][h][:] for query head h uses
 * KV head h / (num_q_heads / num_kv_heads) and attends over positions
 * j < context_lens[s] read through block_tables[s][:].
 * query [num_seqs, num_q_heads, head_dim] in q_dtype; pools in kv_dtype with
 * scales k_scale / v_scale (see gather_sequence); out double, query's shape.
 * Returns 0, or -1 on a malformed argument / table entry.
 * ------------------------------------------------------------------------- */
int oracle_paged_attention_decode_kv(double* out, const void* query, int q_dtype, const void* key_cache,
                                     const void* value_cache, int kv_dtype, double k_scale, double v_scale,
                                     const int32_t* block_tables, const int32_t* context_lens, double scale,
                                     int64_t num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                                     int block_size, int max_blocks_per_seq, int64_t num_blocks) {
    if (!elem_bytes(q_dtype) || q_dtype == ORC_E4M3 || !elem_bytes(kv_dtype) || num_kv_heads <= 0 ||
        num_q_heads % num_kv_heads != 0 || head_dim <= 0 || block_size <= 0)
        return -1;
    int group = num_q_heads / num_kv_heads;
    for (int64_t s = 0; s < num_seqs; ++s) {
        int64_t n = context_lens[s];
        if (n < 0 || n > (int64_t)max_blocks_per_seq * block_size) return -1;
    }
    /* Each (sequence, KV head) pair is independent; with OpenMP the pairs are
     * shared out over the host threads, each output row still computed by one
     * thread in the same order (the result does not depend on the thread count). */
    int64_t pairs = num_seqs * (int64_t)num_kv_heads;
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
    for (int64_t p = 0; p < pairs; ++p) {
        int64_t s = p / num_kv_heads;
        int g = (int)(p % num_kv_heads);
        int64_t n = context_lens[s];
        int64_t cap = n > 0 ? n : 1;
        double* Kc = (double*)malloc(sizeof(double) * cap * head_dim);
        double* Vc = (double*)malloc(sizeof(double) * cap * head_dim);
        double* x = (double*)malloc(sizeof(double) * cap);
        double* qv = (double*)malloc(sizeof(double) * head_dim);
        int rc = (!Kc || !Vc || !x || !qv) ? -1 : 0;
        if (rc == 0)
            rc = gather_sequence(Kc, Vc, key_cache, value_cache, kv_dtype, k_scale, v_scale,
                                 block_tables + s * max_blocks_per_seq, n, g, num_kv_heads, head_dim,
                                 block_size, max_blocks_per_seq, num_blocks);
        for (int hh = 0; hh < group && rc == 0; ++hh) {
            int h = g * group + hh;
            for (int d = 0; d < head_dim; ++d)
                qv[d] = load_elem(query, (s * num_q_heads + h) * (int64_t)head_dim + d, q_dtype);
            attend(out + (s * num_q_heads + h) * (int64_t)head_dim, qv, Kc, Vc, n, head_dim, scale, x);
        }
        free(Kc); free(Vc); free(x); free(qv);
        bad |= rc != 0;
    }
    return bad ? -1 : 0;
}

/* Decode with query and pools of one type (no scaling). */
int oracle_paged_attention_decode(double* out, const void* query, const void* key_cache,
                                  const void* value_cache, int dtype, const int32_t* block_tables,
                                  const int32_t* context_lens, double scale, int64_t num_seqs,
                                  int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                                  int max_blocks_per_seq, int64_t num_blocks) {
    if (dtype == ORC_E4M3) return -1;
    return oracle_paged_attention_decode_kv(out, query, dtype, key_cache, value_cache, dtype, 1.0, 1.0,
                                            block_tables, context_lens, scale, num_seqs, num_q_heads,
                                            num_kv_heads, head_dim, block_size, max_blocks_per_seq, num_blocks);
}

/* ---------------------------------------------------------------------------
 * Chunked prefill ("Chunked Prefill" on the guide page; chunked prefill mixed
 * with decode on the case-study page, section 六).  Chunk r owns query rows
 * [query_start_loc[r], query_start_loc[r+1]) of the packed query
 * [total_q_tokens, num_q_heads, head_dim]; its sequence holds seq_lens[r]
 * cached tokens of which the last n_r are the chunk itself, so the chunk
 * starts at absolute position c0 = seq_lens[r] - n_r.  Row i (absolute
 * position c0 + i) attends causally to keys j <= c0 + i.
 * row_select (may be NULL = all rows) lets a caller evaluate a sample of rows;
 * unselected output rows are left untouched.
 * ------------------------------------------------------------------------- */
int oracle_paged_attention_prefill_chunk_kv(double* out, const void* query, int q_dtype, const void* key_cache,
                                            const void* value_cache, int kv_dtype, double k_scale, double v_scale,
                                            const int32_t* block_tables, const int32_t* seq_lens,
                                            const int32_t* query_start_loc, int num_chunks, double scale,
                                            int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                                            int max_blocks_per_seq, int64_t num_blocks, const uint8_t* row_select) {
    if (!elem_bytes(q_dtype) || q_dtype == ORC_E4M3 || !elem_bytes(kv_dtype) || num_kv_heads <= 0 ||
        num_q_heads % num_kv_heads != 0 || head_dim <= 0 || block_size <= 0)
        return -1;
    int group = num_q_heads / num_kv_heads;
    for (int r = 0; r < num_chunks; ++r) {
        int64_t nq = (int64_t)query_start_loc[r + 1] - query_start_loc[r];
        int64_t len = seq_lens[r];
        if (nq < 0 || len < nq || len > (int64_t)max_blocks_per_seq * block_size) return -1;
    }
    /* (chunk, KV head) pairs are independent: shared out over the host
     * threads under OpenMP, each output row computed by one thread. */
    int64_t pairs = (int64_t)num_chunks * num_kv_heads;
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
    for (int64_t p = 0; p < pairs; ++p) {
        int r = (int)(p / num_kv_heads);
        int g = (int)(p % num_kv_heads);
        int64_t q0 = query_start_loc[r];
        int64_t nq = (int64_t)query_start_loc[r + 1] - q0;
        int64_t len = seq_lens[r];
        int64_t c0 = len - nq;
        int64_t cap = len > 0 ? len : 1;
        double* Kc = (double*)malloc(sizeof(double) * cap * head_dim);
        double* Vc = (double*)malloc(sizeof(double) * cap * head_dim);
        double* x = (double*)malloc(sizeof(double) * cap);
        double* qv = (double*)malloc(sizeof(double) * head_dim);
        int rc = (!Kc || !Vc || !x || !qv) ? -1 : 0;
        if (rc == 0)
            rc = gather_sequence(Kc, Vc, key_cache, value_cache, kv_dtype, k_scale, v_scale,
                                 block_tables + (int64_t)r * max_blocks_per_seq, len, g, num_kv_heads,
                                 head_dim, block_size, max_blocks_per_seq, num_blocks);
        for (int64_t i = 0; i < nq && rc == 0; ++i) {
            int64_t row = q0 + i;
            if (row_select && !row_select[row]) continue;
            for (int hh = 0; hh < group; ++hh) {
                int h = g * group + hh;
                for (int d = 0; d < head_dim; ++d)
                    qv[d] = load_elem(query, (row * num_q_heads + h) * (int64_t)head_dim + d, q_dtype);
                /* causal key set: positions 0 .. c0 + i inclusive */
                attend(out + (row * num_q_heads + h) * (int64_t)head_dim, qv, Kc, Vc, c0 + i + 1,
                       head_dim, scale, x);
            }
        }
        free(Kc); free(Vc); free(x); free(qv);
        bad |= rc != 0;
    }
    return bad ? -1 : 0;
}

/* Prefill with query and pools of one type (no scaling). */
int oracle_paged_attention_prefill_chunk(double* out, const void* query, const void* key_cache,
                                         const void* value_cache, int dtype, const int32_t* block_tables,
                                         const int32_t* seq_lens, const int32_t* query_start_loc,
                                         int num_chunks, double scale, int num_q_heads, int num_kv_heads,
                                         int head_dim, int block_size, int max_blocks_per_seq,
                                         int64_t num_blocks, const uint8_t* row_select) {
    if (dtype == ORC_E4M3) return -1;
    return oracle_paged_attention_prefill_chunk_kv(out, query, dtype, key_cache, value_cache, dtype, 1.0, 1.0,
                                                   block_tables, seq_lens, query_start_loc, num_chunks, scale,
                                                   num_q_heads, num_kv_heads, head_dim, block_size,
                                                   max_blocks_per_seq, num_blocks, row_select);
}
