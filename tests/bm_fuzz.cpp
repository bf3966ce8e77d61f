// Random operation driver for the host block manager, built with the address
// and undefined-behaviour sanitizers by test_block_manager_sanitized.py.  It
// calls every entry point of include/pagedkv_block_manager.h, valid and
// invalid (unknown ids, null or short buffers, swapped-out sequences), and
// checks the pool's conservation laws after each operation:
//   sum of reference counts == total length of the resident block tables,
//   free + evictable + referenced blocks == num_blocks,
//   free host blocks + host blocks held by swapped-out sequences == host pool.
#include <cstdio>
#include <cstdlib>
#include <map>
#include <random>
#include <set>
#include <vector>

#include "pagedkv_block_manager.h"

#define CHECK(c)                                                              \
    do {                                                                      \
        if (!(c)) {                                                           \
            std::fprintf(stderr, "check failed at line %d: %s\n", __LINE__, #c); \
            std::exit(1);                                                     \
        }                                                                     \
    } while (0)

int main(int argc, char** argv) {
    const unsigned seed = argc > 1 ? static_cast<unsigned>(std::atoi(argv[1])) : 1u;
    std::mt19937 rng(seed);
    auto U = [&](int n) { return static_cast<int>(rng() % static_cast<unsigned>(n)); };
    const int B = 1 << (2 + U(3));
    const int64_t NB = 24 + U(40), NH = 16 + U(24);
    pkv_block_manager* bm = pkv_bm_create(NB, B, static_cast<int>(seed & 1));
    CHECK(bm && pkv_bm_create(0, B, 1) == nullptr && pkv_bm_create(NB, 0, 1) == nullptr);
    CHECK(pkv_bm_set_host_blocks(bm, NH) == PKV_BM_OK && pkv_bm_set_host_blocks(bm, -1) == PKV_BM_EINVAL);
    std::map<int64_t, bool> seqs;  // id -> swapped out
    std::map<int64_t, int64_t> host_held;
    int64_t next = 0, swapped_out = 0, swapped_in = 0, cow_pairs = 0;
    std::vector<int64_t> slots(512), pairs(2 * 512);
    std::vector<int32_t> table(512);
    for (int step = 0; step < 4000; ++step) {
        std::vector<int64_t> ids;
        for (auto& kv : seqs) ids.push_back(kv.first);
        const int64_t any = ids.empty() ? 12345 : ids[U(static_cast<int>(ids.size()))];
        const int op = U(10);
        std::vector<int32_t> toks(U(3 * B + 1));
        for (auto& t : toks) t = U(6);  // few distinct ids: prefix hits are common
        int64_t n = 0, done = 0, cached = 0;
        int rc = 0;
        if (op == 0 || ids.empty()) {
            rc = pkv_bm_add_sequence(bm, next, toks.data(), static_cast<int64_t>(toks.size()), &cached);
            CHECK(rc == PKV_BM_OK || rc == PKV_BM_ENOSPACE);
            if (rc == PKV_BM_OK) {
                CHECK(cached % B == 0 && cached <= static_cast<int64_t>(toks.size()));
                seqs[next] = false;
            }
            ++next;
        } else if (op <= 3) {
            rc = pkv_bm_append(bm, any, toks.data(), static_cast<int64_t>(toks.size()), slots.data(), pairs.data(),
                               U(2), &n);
            CHECK(seqs[any] ? rc == PKV_BM_EINVAL : (rc == PKV_BM_OK || rc == PKV_BM_ENOSPACE || rc == PKV_BM_EBUFFER));
            if (rc == PKV_BM_OK) {
                for (size_t i = 0; i < toks.size(); ++i) CHECK(slots[i] >= 0 && slots[i] < NB * B);
                cow_pairs += n;
            }
        } else if (op == 4) {
            std::vector<int64_t> batch;
            for (auto& kv : seqs)
                if (!kv.second) batch.push_back(kv.first);
            std::vector<int32_t> bt(batch.size(), 1);
            rc = pkv_bm_append_batch(bm, batch.data(), bt.data(), static_cast<int64_t>(batch.size()), slots.data(),
                                     pairs.data(), 512, &n, &done);
            CHECK(rc == PKV_BM_OK || rc == PKV_BM_ENOSPACE);
            CHECK(done <= static_cast<int64_t>(batch.size()) && n <= done);
        } else if (op == 5) {
            rc = pkv_bm_fork(bm, any, next);
            CHECK(seqs[any] ? rc == PKV_BM_EINVAL : rc == PKV_BM_OK);
            if (rc == PKV_BM_OK) seqs[next] = false;
            ++next;
        } else if (op == 6) {
            rc = pkv_bm_swap_out(bm, any, pairs.data(), U(2) ? 512 : 1, &n);
            CHECK(seqs[any] ? rc == PKV_BM_EINVAL : (rc == PKV_BM_OK || rc == PKV_BM_ENOSPACE || rc == PKV_BM_EBUFFER));
            if (rc == PKV_BM_OK) {
                ++swapped_out;
                seqs[any] = true;
                host_held[any] = n;
                std::set<int64_t> hs;
                for (int64_t i = 0; i < n; ++i) {
                    CHECK(pairs[2 * i] >= 0 && pairs[2 * i] < NB && pairs[2 * i + 1] >= 0 && pairs[2 * i + 1] < NH);
                    hs.insert(pairs[2 * i + 1]);
                }
                CHECK(static_cast<int64_t>(hs.size()) == n);
            }
        } else if (op == 7) {
            std::vector<int64_t> out_ids;
            for (auto& kv : seqs)
                if (kv.second) out_ids.push_back(kv.first);
            const int64_t target = (!out_ids.empty() && U(4)) ? out_ids[U(static_cast<int>(out_ids.size()))] : any;
            rc = pkv_bm_swap_in(bm, target, pairs.data(), U(4) ? 512 : 0, &n);
            CHECK(!seqs[target] ? rc == PKV_BM_EINVAL
                                : (rc == PKV_BM_OK || rc == PKV_BM_ENOSPACE || rc == PKV_BM_EBUFFER));
            if (rc == PKV_BM_OK) {
                ++swapped_in;
                CHECK(n == host_held[target]);
                std::set<int64_t> ds;
                for (int64_t i = 0; i < n; ++i) {
                    CHECK(pairs[2 * i + 1] >= 0 && pairs[2 * i + 1] < NB && pkv_bm_ref_count(bm, pairs[2 * i + 1]) == 1);
                    ds.insert(pairs[2 * i + 1]);
                }
                CHECK(static_cast<int64_t>(ds.size()) == n);
                seqs[target] = false;
                host_held.erase(target);
            }
        } else if (op == 8) {
            rc = pkv_bm_free(bm, any);
            CHECK(rc == PKV_BM_OK || ids.empty());
            seqs.erase(any);
            host_held.erase(any);
        } else {
            // invalid and edge arguments: nothing may change
            CHECK(pkv_bm_append(nullptr, any, nullptr, 0, nullptr, nullptr, 0, nullptr) == PKV_BM_EINVAL);
            CHECK(pkv_bm_free(bm, -7) == PKV_BM_EINVAL && pkv_bm_fork(bm, any, any) == PKV_BM_EINVAL);
            CHECK(pkv_bm_slots(bm, any, 0, 1 << 20, slots.data()) == PKV_BM_EINVAL);
            CHECK(pkv_bm_ref_count(bm, NB) == PKV_BM_EINVAL && pkv_bm_ref_count(bm, -1) == PKV_BM_EINVAL);
            CHECK(pkv_bm_swap_in(bm, -7, pairs.data(), 512, &n) == PKV_BM_EINVAL);
            int64_t nb = 0;
            rc = pkv_bm_block_table(bm, any, table.data(), 0, &nb);
            CHECK(seqs[any] ? rc == PKV_BM_EINVAL : (nb == 0 ? rc == PKV_BM_OK : rc == PKV_BM_EBUFFER));
        }
        // conservation laws
        int64_t st[9];
        CHECK(pkv_bm_stats(bm, st, 9) == 9);
        int64_t refs = 0, referenced = 0;
        for (int64_t b = 0; b < NB; ++b) {
            const int r = pkv_bm_ref_count(bm, b);
            CHECK(r >= 0);
            refs += r;
            referenced += r > 0;
        }
        int64_t table_len = 0, held = 0;
        for (auto& kv : seqs) {
            CHECK(pkv_bm_num_tokens(bm, kv.first) >= 0);
            if (kv.second) {
                held += host_held[kv.first];
                continue;
            }
            int64_t nb = 0;
            CHECK(pkv_bm_block_table(bm, kv.first, table.data(), 512, &nb) == PKV_BM_OK);
            CHECK(nb == (pkv_bm_num_tokens(bm, kv.first) + B - 1) / B);
            for (int64_t i = 0; i < nb; ++i) CHECK(table[i] >= 0 && table[i] < NB && pkv_bm_ref_count(bm, table[i]) > 0);
            table_len += nb;
        }
        CHECK(refs == table_len);
        CHECK(st[0] + st[1] + referenced == NB);
        CHECK(st[7] + held == NH);
        CHECK(st[6] == static_cast<int64_t>(seqs.size()));
        int64_t out = 0;
        for (auto& kv : seqs) out += kv.second;
        CHECK(st[8] == out);
    }
    pkv_bm_destroy(bm);
    std::fprintf(stderr, "swaps out %lld, in %lld, copy-on-write pairs %lld\n", (long long)swapped_out,
                 (long long)swapped_in, (long long)cow_pairs);
    CHECK(swapped_out >= 20 && swapped_in >= 15 && cow_pairs >= 5);
    std::printf("ok %u\n", seed);
    return 0;
}
