// Random operation driver for the host block manager, built with the address
// and undefined-behaviour sanitizers by test_block_manager_sanitized.py.  It
// calls every entry point of include/pagedkv_block_manager.h, valid and
// invalid (unknown ids, null or short buffers, swapped-out sequences), and
// checks the pool's conservation laws after each operation:
//   sum of reference counts == total length of the resident block tables,
//   free + evictable + referenced blocks == num_blocks,
//   free host blocks + distinct host blocks of swapped-out tables == host pool
// and that group swaps move each distinct block once and rebuild every table.
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
    std::map<int64_t, std::vector<int64_t>> host_table;  // swapped-out sequence -> its host blocks
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
        } else if (op == 6 || op == 7) {
            // a group of 1-3 sequences; mostly of the right state, sometimes any (invalid) id
            const bool out = op == 6;
            std::vector<int64_t> pool_ids;
            for (auto& kv : seqs)
                if (kv.second != out) pool_ids.push_back(kv.first);
            std::vector<int64_t> group;
            const int want = 1 + U(3);
            for (int g = 0; g < want && !pool_ids.empty(); ++g) {
                const int j = U(static_cast<int>(pool_ids.size()));
                group.push_back(pool_ids[j]);
                pool_ids.erase(pool_ids.begin() + j);
            }
            if (group.empty() || U(8) == 0) group.push_back(any);  // possibly wrong state or a repeat
            bool valid = true;
            std::set<int64_t> uniq(group.begin(), group.end());
            if (uniq.size() != group.size()) valid = false;
            for (int64_t g : group)
                if (!seqs.count(g) || seqs[g] != !out) valid = false;
            std::map<int64_t, std::vector<int32_t>> before;
            if (valid && out)
                for (int64_t g : group) {
                    int64_t nb = 0;
                    CHECK(pkv_bm_block_table(bm, g, table.data(), 512, &nb) == PKV_BM_OK);
                    before[g].assign(table.begin(), table.begin() + nb);
                }
            const int64_t cap = U(5) ? 512 : 1;
            rc = out ? pkv_bm_swap_out_group(bm, group.data(), static_cast<int64_t>(group.size()), pairs.data(), cap, &n)
                     : pkv_bm_swap_in_group(bm, group.data(), static_cast<int64_t>(group.size()), pairs.data(), cap, &n);
            if (!valid) {
                CHECK(rc == PKV_BM_EINVAL);
            } else {
                CHECK(rc == PKV_BM_OK || rc == PKV_BM_ENOSPACE || rc == PKV_BM_EBUFFER);
            }
            if (rc == PKV_BM_OK) {
                std::map<int64_t, int64_t> m;  // pair source -> destination, each source once
                std::set<int64_t> dsts;
                for (int64_t i = 0; i < n; ++i) {
                    CHECK(m.emplace(pairs[2 * i], pairs[2 * i + 1]).second && dsts.insert(pairs[2 * i + 1]).second);
                    CHECK(pairs[2 * i + 1] >= 0 && pairs[2 * i + 1] < (out ? NH : NB));
                }
                for (int64_t g : group) {
                    if (out) {
                        std::vector<int64_t> ht;
                        for (int32_t b : before[g]) {
                            CHECK(m.count(b));
                            ht.push_back(m[b]);
                        }
                        host_table[g] = ht;
                        seqs[g] = true;
                        ++swapped_out;
                    } else {
                        int64_t nb = 0;
                        CHECK(pkv_bm_block_table(bm, g, table.data(), 512, &nb) == PKV_BM_OK);
                        CHECK(nb == static_cast<int64_t>(host_table[g].size()));
                        for (int64_t i = 0; i < nb; ++i) CHECK(m.count(host_table[g][i]) && table[i] == m[host_table[g][i]]);
                        host_table.erase(g);
                        seqs[g] = false;
                        ++swapped_in;
                    }
                }
            }
        } else if (op == 8) {
            rc = pkv_bm_free(bm, any);
            CHECK(rc == PKV_BM_OK || ids.empty());
            seqs.erase(any);
            host_table.erase(any);
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
        int64_t table_len = 0;
        std::set<int64_t> held_host;
        for (auto& kv : seqs) {
            CHECK(pkv_bm_num_tokens(bm, kv.first) >= 0);
            if (kv.second) {
                held_host.insert(host_table[kv.first].begin(), host_table[kv.first].end());
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
        CHECK(st[7] + static_cast<int64_t>(held_host.size()) == NH);
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
