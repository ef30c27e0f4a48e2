// tables96.cpp -- host construction of the 96-bit class table (see tables96.h).
#include "tables96.h"

#include <algorithm>
#include <atomic>
#include <cmath>
#include <thread>

#include "tables.h"

namespace llvq {
namespace {

constexpr int kDim = 24;

int popc24(uint32_t w) { return __builtin_popcount(w & 0xFFFFFFu); }

int bitlen128(u128 x) {
    int n = 0;
    while (x) { n++; x >>= 1; }
    return n;
}

// Truncated product of two power series with integer coefficients.
std::vector<__int128> series_mul(const std::vector<__int128> &a, const std::vector<__int128> &b) {
    const size_t n = a.size();
    std::vector<__int128> c(n, 0);
    for (size_t i = 0; i < n; i++) {
        if (!a[i]) continue;
        for (size_t j = 0; i + j < n; j++) c[i + j] += a[i] * b[j];
    }
    return c;
}

// Shell sizes from the theta series of the Leech lattice: theta = E_12 - (65520/691) Delta
// gives N_m = 65520 (sigma_11(m) - tau(m)) / 691 for m >= 1, with Delta(q) = q prod (1 - q^n)^24
// = sum tau(m) q^m.  prod (1 - q^n) comes from Euler's pentagonal number theorem.
bool shell_sizes(int mmax, std::vector<u128> &N, std::string &err) {
    std::vector<__int128> e(mmax + 1, 0);
    for (long j = 0;; j++) {
        const long a = j * (3 * j - 1) / 2, b = j * (3 * j + 1) / 2;
        if (a > mmax) break;
        const int sg = (j & 1) ? -1 : 1;
        e[a] += sg;
        if (j > 0 && b <= mmax) e[b] += sg;
    }
    const std::vector<__int128> e2 = series_mul(e, e), e4 = series_mul(e2, e2), e8 = series_mul(e4, e4);
    const std::vector<__int128> e24 = series_mul(series_mul(e8, e8), e8);
    N.assign(mmax + 1, 0);
    for (int m = 1; m <= mmax; m++) {
        const __int128 tau = e24[m - 1];
        u128 sigma = 0;
        for (int d = 1; d <= m; d++) {
            if (m % d) continue;
            u128 p = 1;
            for (int i = 0; i < 11; i++) p *= (u128)d;
            sigma += p;
        }
        const __int128 num = (__int128)65520 * ((__int128)sigma - tau);
        if (num < 0 || num % 691 != 0) { err = "theta-series shell size not integral"; return false; }
        N[m] = (u128)(num / 691);
    }
    if (N[1] != 0 || N[2] != 196560 || N[3] != 16773120 || N[4] != 398034000) {
        err = "theta-series shell sizes disagree with the known first shells";
        return false;
    }
    return true;
}

// ceil(b 2^128 / P) for b < P <= 2^80: three long-division chunks of at most 47 bits keep the
// shifted remainder below 2^127.
u128 scaled_ratio_up(u128 b, u128 P) {
    u128 q = 0, r = b;
    const int chunks[3] = {47, 47, 34};
    for (int c : chunks) {
        r <<= c;
        const u128 qc = r / P;
        r -= qc * P;
        q = (q << c) | qc;
    }
    return q + (r != 0 ? 1 : 0);
}

// Binomial coefficients C(n, k), n <= 24.
struct Binom {
    uint64_t c[25][25];
    Binom() {
        for (int n = 0; n <= 24; n++)
            for (int k = 0; k <= 24; k++) c[n][k] = k == 0 ? 1 : (n == 0 ? 0 : c[n - 1][k - 1] + (k <= n - 1 ? c[n - 1][k] : 0));
    }
};
const Binom kBinom;

// Classes of one shell in index order: even coset first, then odd; inside a coset the sorted
// magnitude tuples a_0 >= a_1 >= ... >= a_23 in ascending lexicographic order.  The search
// picks the magnitude groups from the largest magnitude down, each magnitude in ascending
// order and, for one magnitude, its count in ascending order (with the same leading groups, a
// smaller count puts a smaller magnitude earlier), so the classes come out in index order.
struct ShellEnum {
    const Tables96 *T = nullptr;
    int m = 0;
    Rec96 *out = nullptr;      // null: count only
    int64_t n = 0;             // valid classes so far
    u128 offset = 0;           // index offset inside the shell (fill mode)
    bool bad = false;
    int64_t n_even = 0;        // classes of the even coset (enumerated first)
    int gv[kDim], gc[kDim], ng = 0;   // groups chosen so far, descending magnitude

    void run() {
        const int norm = 16 * m;
        for (int parity = 0; parity <= 1; parity++) {
            int top = (int)std::sqrt((double)norm) + 1;
            while (top * top > norm) top--;
            if ((top & 1) != parity) top--;
            if (top >= parity) dfs(kDim, norm, top, parity);
            if (parity == 0) n_even = n;
        }
    }

    // left coordinates still to fill with magnitudes in [low, vmax] (same parity), norm rem
    void dfs(int left, int rem, int vmax, int low) {
        for (int v = low; v <= vmax; v += 2) {
            const int sq = v * v;
            if ((long)left * sq < rem) continue;                   // too small to absorb rem
            if (sq > rem && v > low) break;
            for (int c = 1; c <= left; c++) {
                const int r2 = rem - c * sq;
                if (r2 < 0) break;
                const int l2 = left - c;
                gv[ng] = v;
                gc[ng] = c;
                if (l2 == 0) {
                    if (r2 == 0) { ng++; emit(); ng--; }
                    break;
                }
                if (v - 2 < low) continue;                          // nothing smaller to fill with
                if ((long)l2 * (v - 2) * (v - 2) < r2) continue;    // the rest cannot reach r2
                if ((long)l2 * low * low > r2) break;               // the rest cannot be that small
                ng++;
                dfs(l2, r2, v - 2, low);
                ng--;
            }
        }
    }

    void emit() {
        const bool odd = gv[0] & 1;
        int nnz = 0, k = 0, sum_abs = 0, signed_sum = 0;
        for (int g = 0; g < ng; g++) {
            if (gv[g]) nnz += gc[g];
            if (gv[g] % 4 == 2) k += gc[g];
            sum_abs += gv[g] * gc[g];
            signed_sum += (gv[g] % 4 == 3 ? gv[g] : -gv[g]) * gc[g];
        }
        if (!odd) {
            if (T->words_of_weight[k] == 0) return;                // pattern must be a codeword
            if (k == 0 && (sum_abs / 4) % 2 != 0) return;          // sum = 0 (mod 8) impossible
        } else if (((signed_sum % 8) + 8) % 8 != 4) {
            return;                                                // sum with T empty must be 4 (mod 8)
        }
        n++;
        if (!out) return;
        // one list, ascending magnitude: off-codeword groups, then codeword groups (odd: all)
        int lv[kRec96Groups], lc[kRec96Groups], nl = 0, nC = 0;
        u128 PC = 1, PS = 1;
        int leftC = odd ? kDim : kDim - k, leftS = odd ? 0 : k;
        for (int pass = 0; pass < 2; pass++)
            for (int g = ng - 1; g >= 0; g--) {
                const bool onS = !odd && gv[g] % 4 == 2;
                if (onS != (pass == 1)) continue;
                if (nl == kRec96Groups) { bad = true; return; }
                lv[nl] = gv[g];
                lc[nl] = gc[g];
                if (pass == 0) {
                    nC += gc[g];
                    PC *= (u128)kBinom.c[leftC][gc[g]];
                    leftC -= gc[g];
                } else {
                    PS *= (u128)kBinom.c[leftS][gc[g]];
                    leftS -= gc[g];
                }
                nl++;
            }
        const u128 P = PC * PS;
        const uint32_t A = odd ? 4096u : (uint32_t)T->words_of_weight[k];
        const int B = odd ? 0 : (k > 0 ? nnz - 1 : nnz);
        const u128 size = (u128)A * ((u128)1 << B) * P;
        const u128 start = T->shell_start[m] + offset;
        offset += size;
        Rec96 &R = out[n - 1];
        R = Rec96{};
        R.start_lo = (uint64_t)start;
        R.start_hi = (uint32_t)(start >> 64);
        if ((start >> 96) != 0 || P > ((u128)1 << 80) || nC != (odd ? kDim : kDim - k)) bad = true;
        const int t = bitlen128(P - 1);
        const u128 rp = scaled_ratio_up(((u128)1 << t) - P, P);   // R' = ceil(2^(128+t)/P) - 2^128
        R.rcp_lo = (uint64_t)rp;
        R.rcp_hi = (uint64_t)(rp >> 64);
        const uint32_t parity = odd ? 0u : (uint32_t)((sum_abs / 4) & 1);
        R.meta = (uint32_t)t | (uint32_t)m << 7 | (uint32_t)k << 15 | (uint32_t)B << 20 |
                 (odd ? kMeta96Odd : 0u) | (parity ? kMeta96Parity : 0u);
        int cum = 0;
        for (int g = 0; g < kRec96Groups; g++) {
            uint32_t cb = 0x7Fu + 24u, vb = 0u;
            if (g < nl) {
                cum += lc[g];
                cb = 0x7Fu + (uint32_t)cum;
                vb = (uint32_t)lv[g];
            }
            R.cum[g >> 2] |= cb << (8 * (g & 3));
            R.vals[g >> 2] |= vb << (8 * (g & 3));
        }
    }
};

}  // namespace

bool build_tables96(Tables96 &T, int threads, std::string &err) {
    uint32_t words[4096];
    golay_code(words);
    std::copy(words, words + 4096, T.golay_by_mask);
    std::sort(T.golay_by_mask, T.golay_by_mask + 4096);
    std::copy(words, words + 4096, T.golay_by_weight);
    std::sort(T.golay_by_weight, T.golay_by_weight + 4096, [](uint32_t a, uint32_t b) {
        const int wa = popc24(a), wb = popc24(b);
        return wa != wb ? wa < wb : a < b;
    });
    std::fill(T.words_of_weight, T.words_of_weight + 25, 0);
    for (int i = 0; i < 4096; i++) T.words_of_weight[popc24(words[i])]++;
    int acc = 0;
    for (int w = 0; w <= 24; w++) { T.weight_base[w] = acc; acc += T.words_of_weight[w]; }

    std::vector<u128> N;
    if (!shell_sizes(240, N, err)) return false;
    const u128 limit = (u128)1 << 96;
    u128 cum = 0;
    T.shell_start.assign(3, 0);
    T.M = 1;
    for (int m = 2; m < 240; m++) {
        if (cum + N[m] > limit) break;
        T.shell_start[m] = cum;
        cum += N[m];
        T.shell_start.push_back(cum);                 // shell_start[m + 1]
        T.M = m;
    }
    if (T.M < 2 || T.M >= 239) { err = "96-bit shell bound out of range"; return false; }
    T.n_points = cum;

    // classes per shell, counted in parallel (largest shells first)
    T.shell_classes.assign(T.M + 1, 0);
    T.shell_even.assign(T.M + 1, 0);
    std::atomic<int> next(0);
    std::vector<std::thread> pool;
    const int nthreads = std::max(1, threads);
    for (int th = 0; th < nthreads; th++)
        pool.emplace_back([&]() {
            for (;;) {
                const int i = next.fetch_add(1);
                const int m = T.M - i;
                if (m < 2) break;
                ShellEnum e;
                e.T = &T;
                e.m = m;
                e.run();
                T.shell_classes[m] = e.n;
                T.shell_even[m] = e.n_even;
            }
        });
    for (auto &t : pool) t.join();
    T.class_base.assign(T.M + 2, 0);
    int64_t total = 0;
    for (int m = 2; m <= T.M; m++) {
        T.class_base[m] = total;
        total += T.shell_classes[m];
    }
    T.class_base[T.M + 1] = total;
    T.n_classes = total;
    if (total <= 0 || total >= ((int64_t)1 << 32) - 2) { err = "96-bit class count out of range"; return false; }
    return true;
}

bool fill_shell96(const Tables96 &T, int m, Rec96 *out, std::string &err) {
    if (m < 2 || m > T.M) { err = "shell out of range"; return false; }
    ShellEnum e;
    e.T = &T;
    e.m = m;
    e.out = out;
    e.run();
    if (e.bad) { err = "96-bit class outside the record format"; return false; }
    if (e.n != T.shell_classes[m]) { err = "96-bit class count changed between passes"; return false; }
    if (e.offset != T.shell_start[m + 1] - T.shell_start[m]) {
        err = "96-bit class sizes do not add up to the theta-series shell size";
        return false;
    }
    return true;
}

}  // namespace llvq
