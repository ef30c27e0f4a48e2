// tables.cpp -- host construction of the LLVQ index-format tables (see tables.h).
#include "tables.h"

#include <algorithm>
#include <cmath>

namespace llvq {

// Extended Golay code: every multiple a(x) g(x), deg a < 12, of the generator polynomial
// g(x) = 1 + x^2 + x^4 + x^5 + x^6 + x^10 + x^11 of the cyclic [23,12] code (carry-less
// product), with an overall parity bit on coordinate 23.
void golay_code(uint32_t words[4096]) {
    const uint32_t g = 0xC75u;  // bits 0,2,4,5,6,10,11
    for (uint32_t a = 0; a < 4096; a++) {
        uint32_t prod = 0;
        for (int i = 0; i < 12; i++)
            if (a >> i & 1u) prod ^= g << i;
        words[a] = prod | ((uint32_t)(__builtin_popcount(prod & 0xFFFFFFu) & 1) << 23);
    }
}

namespace {

int popc24(uint32_t w) { return __builtin_popcount(w & 0xFFFFFFu); }

u128 factorial(int n) {
    u128 f = 1;
    for (int i = 2; i <= n; i++) f *= (u128)i;
    return f;
}

// Multisets of 24 magnitudes of one parity with sum of squares 16 m, as count vectors over
// the admissible magnitudes (largest magnitude decided first).
struct CountSearch {
    std::vector<int> values;   // admissible magnitudes, descending
    std::vector<int> counts;
    std::vector<std::vector<int>> found;
    void run(size_t vi, int left, int norm) {
        if (vi == values.size()) {
            if (left == 0 && norm == 0) found.push_back(counts);
            return;
        }
        int v = values[vi];
        int sq = v * v;
        int maxn = left;
        if (sq > 0) maxn = std::min(maxn, norm / sq);
        for (int n = maxn; n >= 0; n--) {
            // the smaller magnitudes still to come must be able to absorb the rest
            int rest = norm - n * sq, rest_left = left - n;
            if (vi + 1 < values.size()) {
                int vnext = values[vi + 1];
                if ((long)rest_left * vnext * vnext < rest) continue;
            } else if (rest != 0 || rest_left != 0) {
                continue;
            }
            counts[vi] = n;
            run(vi + 1, rest_left, rest);
            counts[vi] = 0;
        }
    }
};

// Classes of shell m, in the index order: even coset first, then odd; inside a coset by the
// magnitudes sorted descending, compared lexicographically ascending.
void shell_classes(int m, const int words_of_weight[25], std::vector<HostClass> &out) {
    struct Keyed { std::vector<int> key; HostClass c; };
    std::vector<Keyed> all;
    for (int parity = 0; parity <= 1; parity++) {
        CountSearch cs;
        int top = (int)std::sqrt((double)(16 * m)) + 1;
        for (int v = top; v >= 0; v--)
            if ((v & 1) == parity && v * v <= 16 * m) cs.values.push_back(v);
        cs.counts.assign(cs.values.size(), 0);
        cs.run(0, 24, 16 * m);
        for (const auto &cnt : cs.found) {
            HostClass c;
            c.m = m;
            c.odd = parity == 1;
            std::vector<int> key;
            int nnz = 0, k = 0, sum_abs = 0, signed_sum = 0;
            for (size_t i = 0; i < cs.values.size(); i++) {
                int v = cs.values[i], n = cnt[i];
                for (int t = 0; t < n; t++) key.push_back(v);
                if (v != 0) nnz += n;
                if (v % 4 == 2) k += n;
                sum_abs += v * n;
                signed_sum += (v % 4 == 3 ? v : -v) * n;
            }
            c.sum_abs = sum_abs;
            // groups in decode order
            std::vector<std::pair<int, int>> side0, side1;
            for (size_t i = cs.values.size(); i-- > 0;) {          // ascending magnitudes
                if (cnt[i] == 0) continue;
                int v = cs.values[i];
                if (c.odd || v % 4 == 2) side0.push_back({v, cnt[i]});
                else side1.push_back({v, cnt[i]});
            }
            if (!c.odd) {
                if (words_of_weight[k] == 0) continue;                // pattern must be a codeword
                if (k == 0 && (sum_abs / 4) % 2 != 0) continue;        // sum = 0 (mod 8) impossible
                c.k = k;
                c.A = (uint32_t)words_of_weight[k];
                c.B = k > 0 ? nnz - 1 : nnz;
                u128 p0 = factorial(k), p1 = factorial(24 - k);
                for (auto &g : side0) p0 /= factorial(g.second);
                for (auto &g : side1) p1 /= factorial(g.second);
                c.P = p0 * p1;
                c.P_S = p0;
                c.P_C = p1;
            } else {
                int r8 = ((signed_sum % 8) + 8) % 8;                   // sum with T empty
                if (r8 != 4) continue;
                c.A = 4096;
                c.B = 0;
                u128 p = factorial(24);
                for (auto &g : side0) p /= factorial(g.second);
                c.P = p;
                c.P_S = p;
                c.P_C = 1;
            }
            for (auto &g : side0) { c.vals.push_back(g.first); c.cnts.push_back(g.second); }
            for (auto &g : side1) { c.vals.push_back(g.first); c.cnts.push_back(g.second); }
            c.n_side0 = (int)side0.size();
            c.size = (u128)c.A * ((u128)1 << c.B) * c.P;
            all.push_back({key, c});
        }
    }
    std::sort(all.begin(), all.end(), [](const Keyed &a, const Keyed &b) {
        if (a.c.odd != b.c.odd) return !a.c.odd;
        return a.key < b.key;     // descending tuples compared lexicographically
    });
    for (auto &kc : all) out.push_back(kc.c);
}

}  // namespace

bool build_host_tables(int index_bits, HostTables &T, std::string &err) {
    if (index_bits != 48 && index_bits != 72) {
        err = "index_bits must be 48 or 72";
        return false;
    }
    T.index_bits = index_bits;
    uint32_t words[4096];
    golay_code(words);
    std::copy(words, words + 4096, T.golay_by_mask);
    std::sort(T.golay_by_mask, T.golay_by_mask + 4096);
    std::copy(words, words + 4096, T.golay_by_weight);
    std::sort(T.golay_by_weight, T.golay_by_weight + 4096, [](uint32_t a, uint32_t b) {
        int wa = popc24(a), wb = popc24(b);
        return wa != wb ? wa < wb : a < b;
    });
    int words_of_weight[25] = {0};
    for (int i = 0; i < 4096; i++) words_of_weight[popc24(words[i])]++;
    if (words_of_weight[0] != 1 || words_of_weight[8] != 759 || words_of_weight[12] != 2576 ||
        words_of_weight[16] != 759 || words_of_weight[24] != 1) {
        err = "Golay weight distribution check failed";
        return false;
    }
    int acc = 0;
    for (int w = 0; w <= 24; w++) { T.weight_base[w] = acc; acc += words_of_weight[w]; }

    const u128 limit = (u128)1 << index_bits;
    u128 cum = 0;
    T.shell_start.assign(2, 0);
    T.classes.clear();
    for (int m = 2;; m++) {
        std::vector<HostClass> cl;
        shell_classes(m, words_of_weight, cl);
        u128 shell = 0;
        for (auto &c : cl) shell += c.size;
        if (cum + shell > limit) break;
        T.shell_start.push_back(cum);   // shell_start[m]
        for (auto &c : cl) {
            c.start = cum;
            cum += c.size;
            T.classes.push_back(c);
        }
        T.M = m;
        if (m > 400) { err = "shell search did not terminate"; return false; }
    }
    T.shell_start.push_back(cum);       // shell_start[M+1] = N_M
    T.n_points = cum;
    return true;
}

}  // namespace llvq
