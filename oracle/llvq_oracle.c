/*
 * llvq_oracle.c -- plain CPU oracle for LLVQ (Leech lattice vector quantization).
 *
 * TEST INFRASTRUCTURE ONLY: used by the tests, the package smoke check and the bench's
 * CPU-baseline leg, never by the product path.  It shares nothing with the CUDA library.
 *
 * Everything here is written for clarity, not speed: exact unsigned 128-bit integer
 * arithmetic for indices, fp64 for the matrix-vector product, linear scans where a scan
 * is the plainest statement of a step.
 *
 * Page references ("Leech Lattice Vector Quantization for Efficient LLM Compression"):
 *   [notes-K1]  papernotes.org, 方法详解 / 关键设计 1: shells of norm^2 2m, union m = 2..M,
 *               shape-gain split with unit directions x/|x|.
 *   [notes-K2]  papernotes.org, 方法详解 / 关键设计 2: G24 with 4096 codewords; shell by
 *               cumulative offsets; classes = magnitude multiset + even/odd coset, contiguous
 *               ranges; r = I_class mod A, I' = floor(I_class/A), s = I' mod 2^B,
 *               I'' = floor(I'/2^B); r = Golay refinement, s = sign pattern meeting the
 *               congruence check, I'' = lexicographic permutation rank.
 *   [notes-K3]  papernotes.org, 方法详解 / 关键设计 3: Spherical GPTQ (norm-preserving
 *               retraction w^ = (|w| / |w~|) w~, residual propagated through chol(H^-1)^T).
 *   [notes-K4]  papernotes.org, 方法详解 / 关键设计 4: fused dequantize-and-multiply.
 *   [gist-M1]   gist.science, Methodik 1: Leech lattice built from G24, integer vectors in
 *               even and odd cosets, shells of equal squared norm.
 *   [gist-M2]   gist.science, Methodik 2: search over the union of shells, Euclidean distance
 *               (spherical shaping) or cosine similarity (shape-gain); extends Adoul & Barth.
 *   [gist-M3]   gist.science, Methodik 3: index hierarchy shell -> class -> local symmetries.
 * Textbook facts the pages point to but do not print (Conway & Sloane, "Sphere Packings,
 * Lattices and Groups", ch. 4 sec. 11): the sqrt(8)-scaled Leech lattice is the set of
 * integer vectors x with all x_i of one parity, {i : x_i = 2 (mod 4)} (even case) or
 * {i : x_i = 1 (mod 4)} (odd case) a Golay codeword, and sum x_i = 0 (even) or 4 (odd) mod 8.
 */
#include "llvq_oracle.h"

#include <math.h>
#include <pthread.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

typedef unsigned __int128 u128;

#define MAXM 256              /* largest shell any supported budget reaches (96 bits: 214) */

static u128 mk128(uint64_t lo, uint64_t hi) { return ((u128)hi << 64) | lo; }
static void split128(u128 v, uint64_t *lo, uint64_t *hi) {
    *lo = (uint64_t)v;
    *hi = (uint64_t)(v >> 64);
}

/* ===================================================================================== */
/* Extended binary Golay code.  Reading: the cyclic [23,12] Golay code with generator      */
/* polynomial g(x) = 1 + x^2 + x^4 + x^5 + x^6 + x^10 + x^11 (coefficient of x^i on        */
/* coordinate i), extended by an overall parity bit on coordinate 23.  The pages only say  */
/* "extended binary Golay code, 4096 codewords" [notes-K2]; any equivalent code gives an    */
/* isometric lattice, so fixing one is part of the index format.                           */
/* ===================================================================================== */
static int popcount24(uint32_t w) { return __builtin_popcount(w & 0xFFFFFFu); }

static void golay_generate(uint32_t words[4096]) {
    const uint32_t g = (1u << 0) | (1u << 2) | (1u << 4) | (1u << 5) | (1u << 6) | (1u << 10) | (1u << 11);
    uint32_t rows[12];
    for (int i = 0; i < 12; i++) {
        uint32_t w = g << i;                       /* x^i g(x), coordinates 0..22 */
        uint32_t parity = (uint32_t)(popcount24(w) & 1);
        rows[i] = w | (parity << 23);              /* overall parity on coordinate 23 */
    }
    for (uint32_t msg = 0; msg < 4096; msg++) {    /* every combination of the 12 rows */
        uint32_t w = 0;
        for (int i = 0; i < 12; i++)
            if (msg >> i & 1u) w ^= rows[i];
        words[msg] = w;
    }
}

static int cmp_u32(const void *a, const void *b) {
    uint32_t x = *(const uint32_t *)a, y = *(const uint32_t *)b;
    return (x > y) - (x < y);
}
static int cmp_weight_mask(const void *a, const void *b) {
    uint32_t x = *(const uint32_t *)a, y = *(const uint32_t *)b;
    int wx = popcount24(x), wy = popcount24(y);
    if (wx != wy) return wx - wy;
    return (x > y) - (x < y);
}

int ora_golay_by_mask(uint32_t out[4096]) {
    golay_generate(out);
    qsort(out, 4096, sizeof(uint32_t), cmp_u32);
    return 0;
}

int ora_golay_by_weight(uint32_t out[4096], int32_t base[26]) {
    golay_generate(out);
    qsort(out, 4096, sizeof(uint32_t), cmp_weight_mask);
    for (int w = 0; w <= 25; w++) base[w] = 4096;
    for (int i = 4095; i >= 0; i--) base[popcount24(out[i])] = i;
    for (int w = 24; w >= 0; w--)            /* weights with no word point at the next one */
        if (base[w] == 4096 || base[w] > base[w + 1]) base[w] = base[w + 1];
    return 0;
}

static int golay_contains(const uint32_t sorted_by_mask[4096], uint32_t w, int *pos) {
    int lo = 0, hi = 4095;
    while (lo <= hi) {
        int mid = (lo + hi) / 2;
        if (sorted_by_mask[mid] == w) { if (pos) *pos = mid; return 1; }
        if (sorted_by_mask[mid] < w) lo = mid + 1; else hi = mid - 1;
    }
    return 0;
}

/* ===================================================================================== */
/* Lattice membership by the congruences (textbook; [gist-M1] "even and odd cosets").       */
/* ===================================================================================== */
static int mod_pos(int a, int m) { int r = a % m; return r < 0 ? r + m : r; }

static uint32_t g_golay_mask[4096];
static int g_golay_ready = 0;
static void ensure_golay(void) {
    if (!g_golay_ready) { ora_golay_by_mask(g_golay_mask); g_golay_ready = 1; }
}

int ora_in_leech(const int32_t x[ORA_DIM]) {
    ensure_golay();
    int par = mod_pos(x[0], 2);
    int sum = 0;
    uint32_t pattern = 0;
    for (int i = 0; i < ORA_DIM; i++) {
        if (mod_pos(x[i], 2) != par) return 0;                 /* mod 2: one parity */
        sum += x[i];
        int r4 = mod_pos(x[i], 4);
        if (par == 0 && r4 == 2) pattern |= 1u << i;            /* even: the 2 (mod 4) set */
        if (par == 1 && r4 == 1) pattern |= 1u << i;            /* odd:  the 1 (mod 4) set */
    }
    if (!golay_contains(g_golay_mask, pattern, NULL)) return 0;  /* mod 4: a codeword */
    return mod_pos(sum, 8) == (par == 0 ? 0 : 4);                /* mod 8 */
}

/* ===================================================================================== */
/* Shell enumeration by direct search (no class formula): for each coset and each          */
/* codeword, assign coordinates with the prescribed residue mod 4 and check the norm and    */
/* the mod-8 sum.                                                                          */
/* ===================================================================================== */
typedef struct {
    int32_t *out;
    uint64_t cap, n;
    int target_sum8;
    int res[ORA_DIM];        /* required residue mod 4 per coordinate */
    int minrest[ORA_DIM + 1];/* least squared norm the coordinates i.. can take */
    int x[ORA_DIM];
} enum_ctx;

static void enum_rec(enum_ctx *e, int i, int rem, int sum) {
    if (i == ORA_DIM) {
        if (rem == 0 && mod_pos(sum, 8) == e->target_sum8) {
            if (e->out && e->n < e->cap)
                for (int j = 0; j < ORA_DIM; j++) e->out[e->n * ORA_DIM + j] = e->x[j];
            e->n++;
        }
        return;
    }
    int vmax = (int)floor(sqrt((double)rem)) + 1;
    for (int v = -vmax; v <= vmax; v++) {
        if (mod_pos(v, 4) != e->res[i]) continue;
        int r2 = rem - v * v;
        if (r2 < e->minrest[i + 1]) continue;
        e->x[i] = v;
        enum_rec(e, i + 1, r2, sum + v);
    }
}

uint64_t ora_shell_enumerate(int32_t m, int32_t *out, uint64_t cap) {
    ensure_golay();
    enum_ctx e;
    memset(&e, 0, sizeof e);
    e.out = out;
    e.cap = cap;
    for (int odd = 0; odd <= 1; odd++) {
        e.target_sum8 = odd ? 4 : 0;
        for (int w = 0; w < 4096; w++) {
            uint32_t cw = g_golay_mask[w];
            for (int i = 0; i < ORA_DIM; i++) {
                int in = (int)(cw >> i & 1u);
                e.res[i] = odd ? (in ? 1 : 3) : (in ? 2 : 0);
            }
            e.minrest[ORA_DIM] = 0;
            for (int i = ORA_DIM - 1; i >= 0; i--) {
                int least = (e.res[i] == 0) ? 0 : (e.res[i] == 2 ? 4 : 1);
                e.minrest[i] = e.minrest[i + 1] + least;
            }
            enum_rec(&e, 0, 16 * m, 0);
        }
    }
    return e.n;
}

/* Shell sizes by a coordinate-wise dynamic programme.  For a codeword of weight k the     */
/* number of admissible vectors depends only on k, so the count is                        */
/* sum_k (#codewords of weight k) * (DP over k coordinates of one residue class and 24-k   */
/* of the other), tracking the squared norm and the sum mod 8.                             */
int ora_shell_counts_dp(int32_t mmax, uint64_t *lo, uint64_t *hi) {
    if (mmax < 0 || mmax > MAXM) return -1;
    uint32_t words[4096];
    golay_generate(words);
    u128 nk[ORA_DIM + 1];
    memset(nk, 0, sizeof nk);
    for (int i = 0; i < 4096; i++) nk[popcount24(words[i])] += 1;

    const int NMAX = 16 * mmax;
    const int S = (NMAX + 1) * 8;
    u128 *cur = calloc((size_t)S, sizeof(u128));
    u128 *nxt = calloc((size_t)S, sizeof(u128));
    u128 *total = calloc((size_t)(mmax + 1), sizeof(u128));
    if (!cur || !nxt || !total) { free(cur); free(nxt); free(total); return -2; }

    for (int odd = 0; odd <= 1; odd++) {
        for (int k = 0; k <= ORA_DIM; k++) {
            if (nk[k] == 0) continue;
            memset(cur, 0, (size_t)S * sizeof(u128));
            cur[0] = 1;                                      /* norm 0, sum 0 */
            for (int i = 0; i < ORA_DIM; i++) {
                int in = i < k;                              /* first k coordinates: in word */
                int res = odd ? (in ? 1 : 3) : (in ? 2 : 0);
                memset(nxt, 0, (size_t)S * sizeof(u128));
                int vmax = (int)floor(sqrt((double)NMAX)) + 1, nv = 0;
                int vlist[4 * 64];
                for (int v = -vmax; v <= vmax; v++)           /* values with residue res mod 4 */
                    if (mod_pos(v, 4) == res && v * v <= NMAX) vlist[nv++] = v;
                for (int n = 0; n <= NMAX; n++)
                    for (int s = 0; s < 8; s++) {
                        u128 c = cur[n * 8 + s];
                        if (!c) continue;
                        for (int t = 0; t < nv; t++) {
                            int v = vlist[t], n2 = n + v * v;
                            if (n2 > NMAX) continue;
                            nxt[n2 * 8 + mod_pos(s + v, 8)] += c;
                        }
                    }
                u128 *t = cur; cur = nxt; nxt = t;
            }
            for (int m = 0; m <= mmax; m++) total[m] += nk[k] * cur[(16 * m) * 8 + (odd ? 4 : 0)];
        }
    }
    for (int m = 0; m <= mmax; m++) split128(total[m], &lo[m], &hi[m]);
    free(cur); free(nxt); free(total);
    return 0;
}

/* ===================================================================================== */
/* Lexicographic ranking of arrangements of a multiset ([notes-K2]: I'' is the rank of the */
/* coordinate permutation in lexicographic order).  Groups are numbered in ascending       */
/* magnitude; an arrangement is a sequence of group numbers, and sequences compare         */
/* position by position.                                                                   */
/* An even class has two independent coordinate sets (the codeword S carries the 2-mod-4   */
/* magnitudes, its complement the 0-mod-4 ones); each set's sequence is ranked on its own  */
/* and the two ranks form p = p_S + P_S * p_C (the pages do not say how the two sets       */
/* combine; this is the reading the index format fixes).                                   */
/* ===================================================================================== */
static u128 fact128(int n) {
    u128 f = 1;
    for (int i = 2; i <= n; i++) f *= (u128)i;
    return f;
}

/* binomial coefficients C(n, k), n <= 24, by Pascal's rule */
static u128 g_binom[ORA_DIM + 1][ORA_DIM + 1];
static int g_binom_ready = 0;
static void ensure_binom(void) {
    if (g_binom_ready) return;
    for (int n = 0; n <= ORA_DIM; n++) {
        g_binom[n][0] = 1;
        for (int k = 1; k <= n; k++) g_binom[n][k] = g_binom[n - 1][k - 1] + (k < n ? g_binom[n - 1][k] : 0);
    }
    g_binom_ready = 1;
}

/* number of distinct arrangements of a multiset with counts rem[0..ng):
 * n! / prod(c_g!) = C(n, c_0) * C(n - c_0, c_1) * ... */
static u128 multinomial(int ng, const int *rem) {
    int n = 0;
    for (int g = 0; g < ng; g++) n += rem[g];
    u128 r = 1;
    for (int g = 0; g < ng; g++) { r *= g_binom[n][rem[g]]; n -= rem[g]; }
    return r;
}

/* unrank: the p-th arrangement (lexicographic, from 0) of the multiset cnt; n = sum cnt */
static int lex_unrank(int ng, const int *cnt, u128 p, int *seq) {
    int rem[ORA_DIM], n = 0;
    for (int g = 0; g < ng; g++) { rem[g] = cnt[g]; n += cnt[g]; }
    if (p >= multinomial(ng, rem)) return -1;
    for (int i = 0; i < n; i++) {
        int chosen = -1;
        for (int g = 0; g < ng; g++) {                    /* smallest group first */
            if (rem[g] == 0) continue;
            rem[g]--;
            u128 c = multinomial(ng, rem);                /* arrangements that put g at i */
            rem[g]++;
            if (p < c) { chosen = g; break; }
            p -= c;
        }
        if (chosen < 0) return -1;
        seq[i] = chosen;
        rem[chosen]--;
    }
    return 0;
}

/* rank: number of arrangements of cnt that precede seq[0..n) lexicographically */
static int lex_rank(int ng, const int *cnt, int n, const int *seq, u128 *out) {
    int rem[ORA_DIM];
    for (int g = 0; g < ng; g++) rem[g] = cnt[g];
    u128 p = 0;
    for (int i = 0; i < n; i++) {
        int gi = seq[i];
        if (gi < 0 || gi >= ng || rem[gi] == 0) return -1;
        for (int g = 0; g < gi; g++) {                    /* smaller groups at position i */
            if (rem[g] == 0) continue;
            rem[g]--;
            p += multinomial(ng, rem);
            rem[g]++;
        }
        rem[gi]--;
    }
    for (int g = 0; g < ng; g++) if (rem[g]) return -1;
    *out = p;
    return 0;
}

int ora_unrank_arrangement(int32_t nv, const int32_t *cnt, uint64_t lo, uint64_t hi, int32_t *seq) {
    ensure_binom();
    int c[ORA_DIM], s[ORA_DIM];
    int n = 0;
    if (nv < 1 || nv > ORA_DIM) return -1;
    for (int g = 0; g < nv; g++) { c[g] = cnt[g]; n += cnt[g]; }
    if (n > ORA_DIM) return -1;
    if (lex_unrank(nv, c, mk128(lo, hi), s)) return -1;
    for (int i = 0; i < n; i++) seq[i] = s[i];
    return 0;
}

int ora_rank_arrangement(int32_t nv, const int32_t *cnt, int32_t n, const int32_t *seq,
                         uint64_t *lo, uint64_t *hi) {
    ensure_binom();
    int c[ORA_DIM], s[ORA_DIM];
    if (nv < 1 || nv > ORA_DIM || n > ORA_DIM) return -1;
    for (int g = 0; g < nv; g++) c[g] = cnt[g];
    for (int i = 0; i < n; i++) s[i] = seq[i];
    u128 p;
    if (lex_rank(nv, c, n, s, &p)) return -1;
    split128(p, lo, hi);
    return 0;
}

/* ===================================================================================== */
/* Classes ([notes-K2]: a class is a leader's multiset of absolute coordinates together    */
/* with its even/odd coset; classes take contiguous index ranges).  Readings: within a    */
/* shell, even-coset classes come first,                                                  */
/* then odd; inside a coset, classes are ordered by their magnitudes sorted descending,   */
/* compared lexicographically ascending.                                                  */
/*   even: k = #{|x_i| = 2 mod 4} must be a Golay weight (0, 8, 12, 16, 24); when k = 0   */
/*         sum|x_i|/4 must be even.  A = #codewords of weight k, B = #nonzero - [k > 0],  */
/*         P = k!/prod(c_v!, v = 2 mod 4) * (24-k)!/prod(c_v!, v = 0 mod 4).              */
/*   odd:  sum_i (a_i if a_i = 3 mod 4 else -a_i) = 4 mod 8 (the value with T empty; the   */
/*         mod-8 sum does not depend on T).  A = 4096, B = 0, P = 24!/prod(c_v!).          */
/* ===================================================================================== */
typedef struct {
    int16_t m;
    int8_t odd, k, nvals;
    uint8_t vals[ORA_DIM], cnts[ORA_DIM];
    uint16_t A;
    int8_t B;
    u128 P, size, offset;       /* offset: global first index */
} ocls;

typedef void (*class_cb)(void *ctx, const ocls *c);

typedef struct {
    int m, odd, target;
    int a[ORA_DIM];
    const int *nk;          /* codewords per weight */
    class_cb cb;
    void *ctx;
} cenum_ctx;

static void make_class(cenum_ctx *e, ocls *c) {
    /* a[] holds the magnitudes sorted descending */
    memset(c, 0, sizeof *c);
    c->m = (int16_t)e->m;
    c->odd = (int8_t)e->odd;
    int nv = 0;
    for (int i = ORA_DIM - 1; i >= 0; i--) {      /* ascending distinct values */
        if (nv > 0 && c->vals[nv - 1] == e->a[i]) c->cnts[nv - 1]++;
        else { c->vals[nv] = (uint8_t)e->a[i]; c->cnts[nv] = 1; nv++; }
    }
    c->nvals = (int8_t)nv;
}

static int class_valid_and_size(ocls *c, const int *nk) {
    int sumabs = 0, nnz = 0, k = 0;
    for (int g = 0; g < c->nvals; g++) {
        sumabs += c->vals[g] * c->cnts[g];
        if (c->vals[g] != 0) nnz += c->cnts[g];
        if (c->vals[g] % 4 == 2) k += c->cnts[g];
    }
    if (!c->odd) {
        if (nk[k] == 0) return 0;
        if (k == 0 && (sumabs / 4) % 2 != 0) return 0;
        c->k = (int8_t)k;
        c->A = (uint16_t)nk[k];
        c->B = (int8_t)(k > 0 ? nnz - 1 : nnz);
        u128 ps = fact128(k), pc = fact128(ORA_DIM - k);
        for (int g = 0; g < c->nvals; g++) {
            if (c->vals[g] % 4 == 2) ps /= fact128(c->cnts[g]);
            else pc /= fact128(c->cnts[g]);
        }
        c->P = ps * pc;
    } else {
        int s = 0;
        for (int g = 0; g < c->nvals; g++)
            s += (c->vals[g] % 4 == 3 ? 1 : -1) * c->vals[g] * c->cnts[g];
        if (mod_pos(s, 8) != 4) return 0;
        c->k = 0;
        c->A = 4096;
        c->B = 0;
        u128 p = fact128(ORA_DIM);
        for (int g = 0; g < c->nvals; g++) p /= fact128(c->cnts[g]);
        c->P = p;
    }
    c->size = (u128)c->A * ((u128)1 << c->B) * c->P;
    return 1;
}

/* choose a[d] ascending (so descending tuples come out in ascending lexicographic order) */
static void cenum_rec(cenum_ctx *e, int d, int rem, int prev) {
    int low = e->odd ? 1 : 0;
    if (d == ORA_DIM) {
        if (rem != 0) return;
        ocls c;
        make_class(e, &c);
        if (class_valid_and_size(&c, e->nk)) e->cb(e->ctx, &c);
        return;
    }
    int left = ORA_DIM - d;               /* coordinates still to fill, this one included */
    for (int v = low; v <= prev; v += 2) {
        int r2 = rem - v * v;
        if (r2 < (left - 1) * low * low) break;         /* the rest cannot be that small */
        if ((long)left * v * v < rem) continue;          /* the rest cannot reach rem */
        e->a[d] = v;
        cenum_rec(e, d + 1, r2, v);
    }
}

static void enumerate_classes(int m, const int *nk, class_cb cb, void *ctx) {
    cenum_ctx e;
    memset(&e, 0, sizeof e);
    e.m = m;
    e.nk = nk;
    e.cb = cb;
    e.ctx = ctx;
    int top = (int)floor(sqrt((double)(16 * m))) + 1;
    for (int odd = 0; odd <= 1; odd++) {               /* even coset first */
        e.odd = odd;
        int start = top;
        if ((start & 1) != odd) start--;
        cenum_rec(&e, 0, 16 * m, start);
    }
}

/* ===================================================================================== */
/* Codec                                                                                   */
/* ===================================================================================== */
struct ora_codec {
    int bits, M;
    int nk[ORA_DIM + 1];
    uint32_t golay_mask[4096];       /* by mask */
    uint32_t golay_weight[4096];     /* by (weight, mask) */
    int32_t wbase[26];
    u128 shell_off[MAXM + 2];        /* first global index of shell m; shell_off[M+1] = N_M */
    int64_t ncls[MAXM + 1];          /* classes per shell (-1: not built) */
    ocls *cls[MAXM + 1];
    int store_all;                   /* 1: keep every shell's class list */
    int cached;                      /* store_all = 0: the one shell kept after its use (-1: none) */
};

typedef struct { ocls *v; int64_t n, cap; u128 next; } clist;
static void clist_push(void *ctx, const ocls *c) {
    clist *l = ctx;
    if (l->n == l->cap) {
        l->cap = l->cap ? 2 * l->cap : 64;
        l->v = realloc(l->v, (size_t)l->cap * sizeof(ocls));
    }
    l->v[l->n] = *c;
    l->v[l->n].offset = l->next;
    l->next += c->size;
    l->n++;
}

static int build_shell(ora_codec *c, int m) {
    if (c->ncls[m] >= 0) return 0;
    clist l = {0};
    l.next = c->shell_off[m];
    enumerate_classes(m, c->nk, clist_push, &l);
    if (l.next != c->shell_off[m + 1]) {           /* class sums must equal the DP count */
        fprintf(stderr, "oracle: shell %d class sum disagrees with the shell count\n", m);
        free(l.v);
        return -1;
    }
    c->cls[m] = l.v;
    c->ncls[m] = l.n;
    return 0;
}

/* Budgets with shells built on demand keep the shell used last, so that indices of one shell
 * in a row build its class list once. */
static void drop_shell(ora_codec *c, int m) {
    if (c->store_all || c->ncls[m] < 0) return;
    if (c->cached >= 0 && c->cached != m) {
        free(c->cls[c->cached]);
        c->cls[c->cached] = NULL;
        c->ncls[c->cached] = -1;
    }
    c->cached = m;
}

ora_codec *ora_codec_create(int32_t index_bits) {
    if (index_bits != 48 && index_bits != 72 && index_bits != 96) return NULL;
    ora_codec *c = calloc(1, sizeof *c);
    if (!c) return NULL;
    ensure_golay();
    ensure_binom();
    c->bits = index_bits;
    ora_golay_by_mask(c->golay_mask);
    ora_golay_by_weight(c->golay_weight, c->wbase);
    for (int i = 0; i < 4096; i++) c->nk[popcount24(c->golay_mask[i])]++;
    for (int m = 0; m <= MAXM; m++) c->ncls[m] = -1;
    c->cached = -1;

    /* shell sizes far enough to pass 2^index_bits (M = 13, 53, 214 for 48, 72, 96 bits) */
    int mbound = index_bits == 48 ? 20 : (index_bits == 72 ? 64 : 230);
    uint64_t lo[MAXM + 1], hi[MAXM + 1];
    if (ora_shell_counts_dp(mbound, lo, hi)) { free(c); return NULL; }
    u128 limit = (u128)1 << index_bits, cum = 0;
    int M = 1;
    c->shell_off[2] = 0;
    for (int m = 2; m <= mbound; m++) {
        u128 n = mk128(lo[m], hi[m]);
        if (cum + n > limit) break;
        cum += n;
        M = m;
        c->shell_off[m + 1] = cum;
    }
    c->M = M;
    c->store_all = index_bits <= 72;
    if (c->store_all)
        for (int m = 2; m <= M; m++)
            if (build_shell(c, m)) { ora_codec_destroy(c); return NULL; }
    return c;
}

void ora_codec_destroy(ora_codec *c) {
    if (!c) return;
    for (int m = 0; m <= MAXM; m++) free(c->cls[m]);
    free(c);
}

int32_t ora_codec_max_shell(const ora_codec *c) { return c->M; }

void ora_codec_npoints(const ora_codec *c, uint64_t *lo, uint64_t *hi) {
    split128(c->shell_off[c->M + 1], lo, hi);
}

void ora_codec_shell_offset(const ora_codec *c, int32_t m, uint64_t *lo, uint64_t *hi) {
    if (m < 2 || m > c->M + 1) { *lo = *hi = 0; return; }
    split128(c->shell_off[m], lo, hi);
}

int64_t ora_codec_shell_nclasses(ora_codec *c, int32_t m) {
    if (m < 2 || m > c->M) return -1;
    if (build_shell(c, m)) return -1;
    int64_t n = c->ncls[m];
    drop_shell(c, m);
    return n;
}

static void info_from(const ocls *o, ora_class_info *out) {
    memset(out, 0, sizeof *out);
    out->m = o->m;
    out->odd = o->odd;
    out->k = o->k;
    out->nvals = o->nvals;
    for (int g = 0; g < o->nvals; g++) { out->vals[g] = o->vals[g]; out->cnts[g] = o->cnts[g]; }
    out->A = o->A;
    out->B = o->B;
    split128(o->P, &out->P_lo, &out->P_hi);
    split128(o->size, &out->size_lo, &out->size_hi);
    split128(o->offset, &out->offset_lo, &out->offset_hi);
}

int ora_codec_shell_class(ora_codec *c, int32_t m, int64_t j, ora_class_info *out) {
    if (m < 2 || m > c->M) return -1;
    if (build_shell(c, m)) return -1;
    int rc = -1;
    if (j >= 0 && j < c->ncls[m]) { info_from(&c->cls[m][j], out); rc = 0; }
    drop_shell(c, m);
    return rc;
}

/* the class holding global index I (shell by cumulative offsets, then class) */
static int find_class(ora_codec *c, u128 I, ocls *out) {
    if (I >= c->shell_off[c->M + 1]) return -1;
    int m = 2;
    while (!(I < c->shell_off[m + 1])) m++;            /* [notes-K2] shell by cumulative offsets */
    if (build_shell(c, m)) return -1;
    /* classes are contiguous ranges in order: the last class whose offset is <= I */
    int64_t lo = 0, hi = c->ncls[m] - 1;
    while (lo < hi) {
        int64_t mid = (lo + hi + 1) / 2;
        if (c->cls[m][mid].offset <= I) lo = mid; else hi = mid - 1;
    }
    *out = c->cls[m][lo];
    drop_shell(c, m);
    return 0;
}

/* Magnitudes a[0..24) of the p-th arrangement of class o, given its codeword word.
 * odd: p is the lexicographic rank of (a_0, ..., a_23) over the whole multiset.
 * even: p_S = p mod P_S and p_C = floor(p / P_S); p_S ranks the magnitudes on the positions of
 * S (ascending position) among the arrangements of the 2-mod-4 groups, p_C ranks those on the
 * other positions among the arrangements of the 0-mod-4 groups. */
static int class_unrank(const ocls *o, uint32_t word, u128 p, int a[ORA_DIM]) {
    if (o->odd) {
        int cnt[ORA_DIM], seq[ORA_DIM];
        for (int g = 0; g < o->nvals; g++) cnt[g] = o->cnts[g];
        if (lex_unrank(o->nvals, cnt, p, seq)) return -1;
        for (int i = 0; i < ORA_DIM; i++) a[i] = o->vals[seq[i]];
        return 0;
    }
    int vS[ORA_DIM], cS[ORA_DIM], vC[ORA_DIM], cC[ORA_DIM], nS = 0, nC = 0;
    for (int g = 0; g < o->nvals; g++) {          /* ascending magnitude within each set */
        if (o->vals[g] % 4 == 2) { vS[nS] = o->vals[g]; cS[nS++] = o->cnts[g]; }
        else { vC[nC] = o->vals[g]; cC[nC++] = o->cnts[g]; }
    }
    const u128 PS = multinomial(nS, cS);
    int seqS[ORA_DIM], seqC[ORA_DIM];
    if (lex_unrank(nS, cS, p % PS, seqS)) return -1;
    if (lex_unrank(nC, cC, p / PS, seqC)) return -1;
    int iS = 0, iC = 0;
    for (int i = 0; i < ORA_DIM; i++)
        a[i] = (word >> i & 1u) ? vS[seqS[iS++]] : vC[seqC[iC++]];
    return 0;
}

/* inverse of class_unrank: the arrangement rank p of the magnitudes a */
static int class_rank(const ocls *o, uint32_t word, const int a[ORA_DIM], u128 *p) {
    int seq[ORA_DIM];
    if (o->odd) {
        int cnt[ORA_DIM];
        for (int g = 0; g < o->nvals; g++) cnt[g] = o->cnts[g];
        for (int i = 0; i < ORA_DIM; i++) {
            seq[i] = -1;
            for (int g = 0; g < o->nvals; g++) if (o->vals[g] == a[i]) seq[i] = g;
        }
        return lex_rank(o->nvals, cnt, ORA_DIM, seq, p);
    }
    int vS[ORA_DIM], cS[ORA_DIM], vC[ORA_DIM], cC[ORA_DIM], nS = 0, nC = 0;
    for (int g = 0; g < o->nvals; g++) {
        if (o->vals[g] % 4 == 2) { vS[nS] = o->vals[g]; cS[nS++] = o->cnts[g]; }
        else { vC[nC] = o->vals[g]; cC[nC++] = o->cnts[g]; }
    }
    int seqS[ORA_DIM], seqC[ORA_DIM], lS = 0, lC = 0;
    for (int i = 0; i < ORA_DIM; i++) {
        const int inS = (int)(word >> i & 1u);
        const int *v = inS ? vS : vC;
        const int nv = inS ? nS : nC;
        int gi = -1;
        for (int g = 0; g < nv; g++) if (v[g] == a[i]) gi = g;
        if (inS) seqS[lS++] = gi; else seqC[lC++] = gi;
    }
    u128 pS, pC;
    if (lex_rank(nS, cS, lS, seqS, &pS) || lex_rank(nC, cC, lC, seqC, &pC)) return -1;
    *p = pS + multinomial(nS, cS) * pC;
    return 0;
}

/* decode ([notes-K2]): shell -> class -> r, s, I'' by division and remainder, then the
 * codeword, the lexicographic arrangement of the magnitudes and the signs. */
static int decode_one(ora_codec *c, u128 I, int32_t x[ORA_DIM], int *shell) {
    ocls o;
    if (find_class(c, I, &o)) return -1;
    u128 Iclass = I - o.offset;
    u128 r = Iclass % o.A;                       /* r  = I_class mod A           */
    u128 I1 = Iclass / o.A;                      /* I' = floor(I_class / A)      */
    u128 s = I1 % ((u128)1 << o.B);              /* s  = I' mod 2^B              */
    u128 p = I1 / ((u128)1 << o.B);              /* I''= floor(I' / 2^B)         */

    uint32_t word;
    if (o.odd) word = c->golay_mask[(int)r];                 /* T: r-th codeword by mask */
    else word = c->golay_weight[c->wbase[o.k] + (int)r];     /* S: r-th word of weight k */

    int a[ORA_DIM];
    if (class_unrank(&o, word, p, a)) return -1;

    if (o.odd) {
        /* x_i = 1 (mod 4) exactly on T */
        for (int i = 0; i < ORA_DIM; i++) {
            int inT = (int)(word >> i & 1u);
            x[i] = (inT == (a[i] % 4 == 1)) ? a[i] : -a[i];
        }
    } else {
        /* bit j of s -> j-th nonzero coordinate (ascending), skipping the highest coordinate
         * of S, which takes the sign that makes #negatives on S = sum|x|/4 (mod 2) */
        int top = -1;
        if (o.k > 0) for (int i = 0; i < ORA_DIM; i++) if (word >> i & 1u) top = i;
        int j = 0, negS = 0, sumabs = 0;
        for (int i = 0; i < ORA_DIM; i++) {
            sumabs += a[i];
            x[i] = a[i];
            if (a[i] == 0 || i == top) continue;
            if ((s >> j) & 1) { x[i] = -a[i]; if (word >> i & 1u) negS++; }
            j++;
        }
        if (top >= 0 && (negS & 1) != ((sumabs / 4) & 1)) x[top] = -a[top];
    }
    if (shell) *shell = o.m;
    return 0;
}

int ora_decode(ora_codec *c, uint64_t lo, uint64_t hi, int32_t x[ORA_DIM]) {
    return decode_one(c, mk128(lo, hi), x, NULL);
}

static int cmp_int_desc(const void *a, const void *b) {
    int x = *(const int *)a, y = *(const int *)b;
    return (x < y) - (x > y);
}

/* encode: the inverse of decode, step by step */
int ora_encode(ora_codec *c, const int32_t x[ORA_DIM], uint64_t *lo, uint64_t *hi) {
    if (!ora_in_leech(x)) return -1;
    int nrm = 0, a[ORA_DIM], sorted[ORA_DIM];
    for (int i = 0; i < ORA_DIM; i++) {
        a[i] = x[i] < 0 ? -x[i] : x[i];
        nrm += a[i] * a[i];
        sorted[i] = a[i];
    }
    if (nrm % 16) return -1;
    int m = nrm / 16;
    if (m < 2 || m > c->M) return -1;
    qsort(sorted, ORA_DIM, sizeof(int), cmp_int_desc);
    if (build_shell(c, m)) return -1;
    int odd = a[0] & 1;
    /* locate the class by its magnitudes and coset */
    int64_t found = -1;
    for (int64_t j = 0; j < c->ncls[m] && found < 0; j++) {
        const ocls *o = &c->cls[m][j];
        if (o->odd != odd) continue;
        int idx = 0, same = 1;
        for (int g = o->nvals - 1; g >= 0 && same; g--)
            for (int t = 0; t < o->cnts[g]; t++)
                if (sorted[idx++] != o->vals[g]) { same = 0; break; }
        if (same) found = j;
    }
    if (found < 0) { drop_shell(c, m); return -1; }
    ocls o = c->cls[m][found];
    drop_shell(c, m);

    uint32_t word = 0;
    for (int i = 0; i < ORA_DIM; i++) {
        if (odd && mod_pos(x[i], 4) == 1) word |= 1u << i;
        if (!odd && a[i] % 4 == 2) word |= 1u << i;
    }
    u128 r = 0;
    if (odd) {
        int pos;
        if (!golay_contains(c->golay_mask, word, &pos)) return -1;
        r = (u128)pos;
    } else {
        int found_r = -1;
        for (int t = c->wbase[o.k]; t < c->wbase[o.k + 1]; t++)
            if (c->golay_weight[t] == word) { found_r = t - c->wbase[o.k]; break; }
        if (found_r < 0) return -1;
        r = (u128)found_r;
    }
    u128 s = 0;
    if (!odd) {
        int top = -1;
        if (o.k > 0) for (int i = 0; i < ORA_DIM; i++) if (word >> i & 1u) top = i;
        int j = 0;
        for (int i = 0; i < ORA_DIM; i++) {
            if (a[i] == 0 || i == top) continue;
            if (x[i] < 0) s |= (u128)1 << j;
            j++;
        }
    }
    u128 p;
    if (class_rank(&o, word, a, &p)) return -1;
    u128 I = o.offset + r + (u128)o.A * (s + ((u128)1 << o.B) * p);
    split128(I, lo, hi);
    return 0;
}

/* Decodes in ascending index order (the results land at their original positions), so a
 * budget with shells built on demand builds each shell once. */
typedef struct { u128 I; int64_t pos; } idx_pos;
static int cmp_idx_pos(const void *a, const void *b) {
    const u128 x = ((const idx_pos *)a)->I, y = ((const idx_pos *)b)->I;
    return x < y ? -1 : (x > y ? 1 : 0);
}

static int64_t decode_sorted(ora_codec *c, int64_t n, const u128 *idx, int8_t *out, int32_t *shell) {
    idx_pos *o = malloc((size_t)(n > 0 ? n : 1) * sizeof(idx_pos));
    if (!o) return -1;
    for (int64_t t = 0; t < n; t++) { o[t].I = idx[t]; o[t].pos = t; }
    if (!c->store_all) qsort(o, (size_t)n, sizeof(idx_pos), cmp_idx_pos);
    int64_t bad = 0;
    for (int64_t u = 0; u < n; u++) {
        int32_t x[ORA_DIM];
        int m = 0;
        const int64_t t = o[u].pos;
        if (decode_one(c, o[u].I, x, &m)) {
            memset(x, 0, sizeof x);
            m = 0;
            bad++;
        }
        for (int i = 0; i < ORA_DIM; i++) out[t * ORA_DIM + i] = (int8_t)x[i];
        if (shell) shell[t] = m;
    }
    free(o);
    return bad;
}

int64_t ora_decode_batch_shell(ora_codec *c, int64_t n, const uint64_t *lo, const uint64_t *hi,
                               int8_t *out, int32_t *shell) {
    u128 *idx = malloc((size_t)(n > 0 ? n : 1) * sizeof(u128));
    if (!idx) return -1;
    for (int64_t t = 0; t < n; t++) idx[t] = mk128(lo[t], hi ? hi[t] : 0);
    const int64_t bad = decode_sorted(c, n, idx, out, shell);
    free(idx);
    return bad;
}

int64_t ora_decode_batch(ora_codec *c, int64_t n, const uint64_t *lo, const uint64_t *hi,
                         int8_t *out) {
    return ora_decode_batch_shell(c, n, lo, hi, out, NULL);
}

/* ===================================================================================== */
/* fp16 -> fp64 (IEEE binary16, exact)                                                   */
/* ===================================================================================== */
double ora_half_to_double(uint16_t h) {
    int sign = h >> 15, e = (h >> 10) & 0x1F, f = h & 0x3FF;
    double v;
    if (e == 0) v = ldexp((double)f, -24);                        /* subnormal */
    else if (e == 31) v = f ? NAN : INFINITY;
    else v = ldexp((double)(f | 0x400), e - 25);
    return sign ? -v : v;
}

/* ===================================================================================== */
/* GEMV / small-batch GEMM in fp64 ([notes-K4]: each block's 24-dim integer vector is      */
/* scaled by its gain and dotted with the activations; [notes-K1]: shape-gain, the        */
/* direction is v/|v| and the gain a scalar).                                            */
/* ===================================================================================== */
static void unpack_word(const uint8_t *wp, int word_bytes, int bits, u128 *index, int *code) {
    uint64_t lo, hi = 0;
    memcpy(&lo, wp, 8);
    if (word_bytes == 16) memcpy(&hi, wp + 8, 8);
    u128 w = mk128(lo, hi);
    *index = w & (((u128)1 << bits) - 1);
    *code = (int)((w >> bits) & 0xFF);
}

typedef struct {
    const ora_codec *c;
    int32_t rows, nb, word_bytes, gain_mode, batch;
    const void *words;
    int64_t pitch;
    const uint16_t *gains, *x;
    double *y;
    int32_t r0, r1;
    int64_t bad;
    const int8_t *vecs;            /* on-demand budgets: every block decoded beforehand */
    const int32_t *shells;         /* (shell 0 = bad index) */
} gemm_job;

static void gemm_rows(gemm_job *J) {
    /* each worker keeps private class lists when shells are built on demand */
    ora_codec *c = (ora_codec *)J->c;
    const uint8_t *W = J->words;
    int64_t K = (int64_t)J->nb * ORA_DIM;
    for (int32_t r = J->r0; r < J->r1; r++) {
        for (int32_t b = 0; b < J->batch; b++) J->y[(int64_t)b * J->rows + r] = 0.0;
        for (int32_t j = 0; j < J->nb; j++) {
            u128 I;
            int code, m = 0;
            unpack_word(W + ((int64_t)r * J->pitch + j) * J->word_bytes, J->word_bytes, c->bits, &I,
                        &code);
            int32_t v[ORA_DIM];
            if (J->vecs) {
                const int64_t blk = (int64_t)r * J->nb + j;
                m = J->shells[blk];
                if (m == 0) { J->bad++; continue; }
                for (int t = 0; t < ORA_DIM; t++) v[t] = J->vecs[blk * ORA_DIM + t];
            } else if (decode_one(c, I, v, &m)) {
                J->bad++;
                continue;
            }
            double scale;
            if (J->gain_mode == 0) scale = ora_half_to_double(J->gains[(int64_t)r * J->nb + j]);
            else scale = ora_half_to_double(J->gains[(int64_t)r * 256 + code]) / (4.0 * sqrt((double)m));
            for (int32_t b = 0; b < J->batch; b++) {
                const uint16_t *xb = J->x + (int64_t)b * K + (int64_t)j * ORA_DIM;
                double acc = 0.0;
                for (int t = 0; t < ORA_DIM; t++) acc += (scale * (double)v[t]) * ora_half_to_double(xb[t]);
                J->y[(int64_t)b * J->rows + r] += acc;
            }
        }
    }
}

/* On-demand budgets (96 bits): decode every block first, in ascending index order. */
static int predecode(ora_codec *c, int32_t rows, int32_t nb, const void *words, int32_t word_bytes,
                     int64_t pitch, int8_t **vecs, int32_t **shells) {
    const int64_t n = (int64_t)rows * nb;
    u128 *idx = malloc((size_t)(n > 0 ? n : 1) * sizeof(u128));
    *vecs = malloc((size_t)(n > 0 ? n : 1) * ORA_DIM);
    *shells = malloc((size_t)(n > 0 ? n : 1) * sizeof(int32_t));
    if (!idx || !*vecs || !*shells) { free(idx); return -1; }
    for (int32_t r = 0; r < rows; r++)
        for (int32_t j = 0; j < nb; j++) {
            int code;
            unpack_word((const uint8_t *)words + ((int64_t)r * pitch + j) * word_bytes, word_bytes, c->bits,
                        &idx[(int64_t)r * nb + j], &code);
        }
    decode_sorted(c, n, idx, *vecs, *shells);
    free(idx);
    return 0;
}

int64_t ora_gemm(ora_codec *c, int32_t rows, int32_t nb, const void *words, int32_t word_bytes,
                 int64_t row_pitch_words, int32_t gain_mode, const uint16_t *gains,
                 const uint16_t *x, int32_t batch, double *y) {
    if ((c->bits == 48) != (word_bytes == 8)) return -1;
    gemm_job J = {c, rows, nb, word_bytes, gain_mode, batch, words, row_pitch_words, gains, x, y,
                  0, rows, 0, NULL, NULL};
    int8_t *vecs = NULL;
    int32_t *shells = NULL;
    if (!c->store_all) {
        if (predecode(c, rows, nb, words, word_bytes, row_pitch_words, &vecs, &shells)) return -1;
        J.vecs = vecs;
        J.shells = shells;
    }
    gemm_rows(&J);
    free(vecs);
    free(shells);
    return J.bad;
}

static void *gemm_thread(void *arg) { gemm_rows((gemm_job *)arg); return NULL; }

int64_t ora_gemm_mt(const ora_codec *c, int32_t rows, int32_t nb, const void *words,
                    int32_t word_bytes, int64_t row_pitch_words, int32_t gain_mode,
                    const uint16_t *gains, const uint16_t *x, int32_t batch, double *y,
                    int32_t nthreads) {
    if ((c->bits == 48) != (word_bytes == 8)) return -1;
    if (!c->store_all)                   /* on-demand shell lists are not shared safely */
        return ora_gemm((ora_codec *)c, rows, nb, words, word_bytes, row_pitch_words, gain_mode, gains, x,
                        batch, y);
    if (nthreads < 1) nthreads = 1;
    if (nthreads > rows) nthreads = rows > 0 ? rows : 1;
    gemm_job *jobs = calloc((size_t)nthreads, sizeof(gemm_job));
    pthread_t *th = calloc((size_t)nthreads, sizeof(pthread_t));
    for (int t = 0; t < nthreads; t++) {
        gemm_job J = {c, rows, nb, word_bytes, gain_mode, batch, words, row_pitch_words, gains, x, y,
                      (int32_t)((int64_t)rows * t / nthreads), (int32_t)((int64_t)rows * (t + 1) / nthreads), 0,
                      NULL, NULL};
        jobs[t] = J;
        pthread_create(&th[t], NULL, gemm_thread, &jobs[t]);
    }
    int64_t bad = 0;
    for (int t = 0; t < nthreads; t++) { pthread_join(th[t], NULL); bad += jobs[t].bad; }
    free(jobs);
    free(th);
    return bad;
}

/* ===================================================================================== */
/* Exhaustive self-checks over whole shells (threads split the codewords).                */
/* ===================================================================================== */
typedef struct {
    ora_codec *c;
    int m_lo, m_hi, tid, nthreads;
    uint64_t *bitmap;              /* one bit per index of shells m_lo..m_hi */
    u128 base;                     /* first index of shell m_lo */
    int64_t points, bad_encode, bad_range, dup, bad_roundtrip, bad_norm;
} check_job;

static void check_point(check_job *J, const int *x, int m) {
    int32_t xx[ORA_DIM];
    for (int i = 0; i < ORA_DIM; i++) xx[i] = x[i];
    uint64_t lo, hi;
    J->points++;
    if (ora_encode(J->c, xx, &lo, &hi)) { J->bad_encode++; return; }
    u128 I = mk128(lo, hi);
    if (I < J->c->shell_off[m] || I >= J->c->shell_off[m + 1]) { J->bad_range++; return; }
    u128 rel = I - J->base;
    uint64_t bit = 1ull << (uint64_t)(rel % 64);
    uint64_t old = __atomic_fetch_or(&J->bitmap[(size_t)(rel / 64)], bit, __ATOMIC_RELAXED);
    if (old & bit) J->dup++;
    int32_t y[ORA_DIM];
    int shell = 0;
    if (decode_one(J->c, I, y, &shell)) { J->bad_roundtrip++; return; }
    int nrm = 0;
    for (int i = 0; i < ORA_DIM; i++) { if (y[i] != xx[i]) { J->bad_roundtrip++; return; } nrm += y[i] * y[i]; }
    if (nrm != 16 * m || shell != m || !ora_in_leech(y)) J->bad_norm++;
}

static void check_rec(check_job *J, enum_ctx *e, int i, int rem, int sum, int m) {
    if (i == ORA_DIM) {
        if (rem == 0 && mod_pos(sum, 8) == e->target_sum8) check_point(J, e->x, m);
        return;
    }
    int vmax = (int)floor(sqrt((double)rem)) + 1;
    for (int v = -vmax; v <= vmax; v++) {
        if (mod_pos(v, 4) != e->res[i]) continue;
        int r2 = rem - v * v;
        if (r2 < e->minrest[i + 1]) continue;
        e->x[i] = v;
        check_rec(J, e, i + 1, r2, sum + v, m);
    }
}

static void *check_thread(void *arg) {
    check_job *J = arg;
    enum_ctx e;
    memset(&e, 0, sizeof e);
    for (int m = J->m_lo; m <= J->m_hi; m++)
        for (int odd = 0; odd <= 1; odd++) {
            e.target_sum8 = odd ? 4 : 0;
            for (int w = J->tid; w < 4096; w += J->nthreads) {
                uint32_t cw = g_golay_mask[w];
                for (int i = 0; i < ORA_DIM; i++) {
                    int in = (int)(cw >> i & 1u);
                    e.res[i] = odd ? (in ? 1 : 3) : (in ? 2 : 0);
                }
                e.minrest[ORA_DIM] = 0;
                for (int i = ORA_DIM - 1; i >= 0; i--)
                    e.minrest[i] = e.minrest[i + 1] + (e.res[i] == 0 ? 0 : (e.res[i] == 2 ? 4 : 1));
                check_rec(J, &e, 0, 16 * m, 0, m);
            }
        }
    return NULL;
}

/* Enumerate every point of shells m_lo..m_hi by direct search, encode it, require the
 * index to fall in its shell's range and to be hit exactly once, and require decode to
 * give the point back (with the right norm and lattice membership).  result[0..6] =
 * points, bad encodes, out-of-range, duplicates, bad round trips, bad norms, indices of
 * the range never hit.  Returns 0 when every count but result[0] is zero. */
int ora_check_shells(ora_codec *c, int32_t m_lo, int32_t m_hi, int32_t nthreads, int64_t result[7]) {
    if (!c->store_all || m_lo < 2 || m_hi > c->M || m_lo > m_hi) return -1;
    if (nthreads < 1) nthreads = 1;
    u128 base = c->shell_off[m_lo], span = c->shell_off[m_hi + 1] - base;
    size_t words = (size_t)((span + 63) / 64);
    uint64_t *bm = calloc(words, sizeof(uint64_t));
    check_job *jobs = calloc((size_t)nthreads, sizeof(check_job));
    pthread_t *th = calloc((size_t)nthreads, sizeof(pthread_t));
    if (!bm || !jobs || !th) { free(bm); free(jobs); free(th); return -2; }
    for (int t = 0; t < nthreads; t++) {
        jobs[t].c = c; jobs[t].m_lo = m_lo; jobs[t].m_hi = m_hi; jobs[t].tid = t;
        jobs[t].nthreads = nthreads; jobs[t].bitmap = bm; jobs[t].base = base;
        pthread_create(&th[t], NULL, check_thread, &jobs[t]);
    }
    for (int k = 0; k < 7; k++) result[k] = 0;
    for (int t = 0; t < nthreads; t++) {
        pthread_join(th[t], NULL);
        result[0] += jobs[t].points; result[1] += jobs[t].bad_encode; result[2] += jobs[t].bad_range;
        result[3] += jobs[t].dup; result[4] += jobs[t].bad_roundtrip; result[5] += jobs[t].bad_norm;
    }
    int64_t missing = 0;
    for (u128 i = 0; i < span; i++)
        if (!(bm[(size_t)(i / 64)] >> (uint64_t)(i % 64) & 1ull)) missing++;
    result[6] = missing;
    free(bm); free(jobs); free(th);
    for (int k = 1; k < 7; k++) if (result[k]) return 1;
    return 0;
}

/* ===================================================================================== */
/* Nearest-point search over the shell union Lambda24(M) = Shell(2) u ... u Shell(M)     */
/* ([notes-K1] 关键设计 1 "多壳层球面与角度搜索": the union of shells, the unit-vector      */
/* inner product for the shape of a shape-gain split; [gist-M2] Methodik 2: two modes,     */
/* Euclidean distance for spherical shaping, cosine similarity for shape-gain, both over   */
/* the union; the search extends Adoul & Barth's single-shell search).                     */
/*                                                                                         */
/* Readings (the pages name the two criteria but print no algorithm):                     */
/*   angular   (mode 0): maximize <y, v> / |v| over v in the union.                        */
/*   Euclidean (mode 1): the reconstruction is c v for a given scale c > 0; minimize       */
/*                       |y - c v|^2, i.e. maximize 2 c <y, v> - c^2 |v|^2.                */
/* Every point of a class has the same norm, so each criterion is the best <y, v> inside   */
/* each class, compared across classes.  Inside a class and for one Golay codeword (the    */
/* 2-mod-4 set S of an even point, the 1-mod-4 set T of an odd one) the best point follows */
/* from the rearrangement inequality (larger |y_i| take larger magnitudes):               */
/*   even: S takes the 2-mod-4 magnitudes and the other positions the 0-mod-4 ones, each   */
/*         in descending order of |y_i|, signs those of y; when the coordinate sum is not  */
/*         0 mod 8 the sign on S with the smallest |y_i| turns (one turn costs least).    */
/*   odd:  the signs follow from T and the magnitudes (x_i = 1 mod 4 exactly on T), so a   */
/*         position wants a 1-mod-4 magnitude when (i in T) equals (y_i >= 0) and a       */
/*         3-mod-4 one otherwise.  Each set takes its own magnitudes in descending order;  */
/*         when a set has more positions than magnitudes of its kind, its smallest-|y|     */
/*         positions take the other kind's smallest magnitudes with the wrong sign, the   */
/*         largest of those |y_i| taking the smallest magnitude.                          */
/* The brute-force search below enumerates the shells from the congruences alone and pins  */
/* these rules on shells 2..4.  Ties keep the first best in the order shell, class,       */
/* codeword (by mask).                                                                     */
/* ===================================================================================== */

/* positions by |y_i| descending, equal values by position */
static void order_desc(const double y[ORA_DIM], int ord[ORA_DIM]) {
    for (int i = 0; i < ORA_DIM; i++) ord[i] = i;
    for (int i = 1; i < ORA_DIM; i++)                     /* insertion sort, stable */
        for (int j = i; j > 0 && fabs(y[ord[j]]) > fabs(y[ord[j - 1]]); j--) {
            int t = ord[j]; ord[j] = ord[j - 1]; ord[j - 1] = t;
        }
}

/* class magnitudes of residue res (mod 4), descending; returns how many */
static int class_mags(const ocls *o, int res, int out[ORA_DIM]) {
    int n = 0;
    for (int g = o->nvals - 1; g >= 0; g--)
        if (o->vals[g] % 4 == res)
            for (int t = 0; t < o->cnts[g]; t++) out[n++] = o->vals[g];
    return n;
}

/* the point of odd class o whose 1-mod-4 set is T with the largest <y, v> */
static void best_odd(const ocls *o, uint32_t T, const double y[ORA_DIM], const int ord[ORA_DIM],
                     int v[ORA_DIM]) {
    int L1[ORA_DIM], L3[ORA_DIM], P1[ORA_DIM], P3[ORA_DIM], a[ORA_DIM];
    int n1 = class_mags(o, 1, L1), n3 = class_mags(o, 3, L3), p1 = 0, p3 = 0;
    for (int t = 0; t < ORA_DIM; t++) {
        int i = ord[t];
        int inT = (int)(T >> i & 1u), pos = y[i] >= 0.0;
        if (inT == pos) P1[p1++] = i; else P3[p3++] = i;
    }
    if (p1 >= n1) {                     /* P1 has s = p1 - n1 positions too many */
        int s = p1 - n1;
        for (int j = 0; j < n1; j++) a[P1[j]] = L1[j];
        for (int j = 0; j < p3; j++) a[P3[j]] = L3[j];
        for (int j = 0; j < s; j++) a[P1[n1 + j]] = L3[n3 - 1 - j];
    } else {                            /* P3 has s = p3 - n3 positions too many */
        int s = p3 - n3;
        for (int j = 0; j < n3; j++) a[P3[j]] = L3[j];
        for (int j = 0; j < p1; j++) a[P1[j]] = L1[j];
        for (int j = 0; j < s; j++) a[P3[n3 + j]] = L1[n1 - 1 - j];
    }
    for (int i = 0; i < ORA_DIM; i++)
        v[i] = ((a[i] % 4 == 1) == (int)(T >> i & 1u)) ? a[i] : -a[i];
}

/* the point of even class o whose 2-mod-4 set is S with the largest <y, v> */
static void best_even(const ocls *o, uint32_t S, const double y[ORA_DIM], const int ord[ORA_DIM],
                      int v[ORA_DIM]) {
    int L2[ORA_DIM], L0[ORA_DIM];
    class_mags(o, 2, L2);
    class_mags(o, 0, L0);
    int j2 = 0, j0 = 0, sum = 0, last_on_S = -1;
    for (int t = 0; t < ORA_DIM; t++) {
        int i = ord[t];
        int a = (S >> i & 1u) ? L2[j2++] : L0[j0++];
        if (S >> i & 1u) last_on_S = i;
        v[i] = y[i] >= 0.0 ? a : -a;
        sum += v[i];
    }
    if (mod_pos(sum, 8) != 0 && last_on_S >= 0) v[last_on_S] = -v[last_on_S];
}

static double dot24(const double y[ORA_DIM], const int v[ORA_DIM]) {
    double s = 0.0;
    for (int i = 0; i < ORA_DIM; i++) s += y[i] * (double)v[i];
    return s;
}

static double search_objective(int mode, double scale, double dot, int norm2) {
    return mode == 0 ? dot / sqrt((double)norm2) : 2.0 * scale * dot - scale * scale * (double)norm2;
}

int ora_search(ora_codec *c, int32_t m_max, int32_t mode, double scale, const double y[ORA_DIM],
               int32_t v_out[ORA_DIM], double *dot_out) {
    if (m_max < 2 || m_max > c->M || (mode != 0 && mode != 1) || (mode == 1 && !(scale > 0.0)))
        return -1;
    int ord[ORA_DIM], v[ORA_DIM];
    order_desc(y, ord);
    double best = -INFINITY, best_dot = 0.0;
    int have = 0;
    for (int m = 2; m <= m_max; m++) {
        if (build_shell(c, m)) return -1;
        for (int64_t j = 0; j < c->ncls[m]; j++) {
            const ocls *o = &c->cls[m][j];
            int first = o->odd ? 0 : c->wbase[o->k], end = o->odd ? 4096 : c->wbase[o->k + 1];
            for (int w = first; w < end; w++) {
                if (o->odd) best_odd(o, c->golay_mask[w], y, ord, v);
                else best_even(o, c->golay_weight[w], y, ord, v);
                double d = dot24(y, v);
                double f = search_objective(mode, scale, d, 16 * m);
                if (!have || f > best) {
                    have = 1; best = f; best_dot = d;
                    for (int i = 0; i < ORA_DIM; i++) v_out[i] = v[i];
                }
            }
        }
        drop_shell(c, m);
    }
    if (dot_out) *dot_out = best_dot;
    return 0;
}

typedef struct {
    ora_codec *c;
    int m_max, mode, tid, nthreads, bad;
    double scale;
    int64_t n;
    const float *X;
    int8_t *V;
    double *dot;
} search_job;

static void *search_thread(void *arg) {
    search_job *j = arg;
    double y[ORA_DIM], d;
    int32_t v[ORA_DIM];
    for (int64_t r = j->tid; r < j->n; r += j->nthreads) {
        for (int i = 0; i < ORA_DIM; i++) y[i] = (double)j->X[r * ORA_DIM + i];
        if (ora_search(j->c, j->m_max, j->mode, j->scale, y, v, &d)) { j->bad = 1; return NULL; }
        for (int i = 0; i < ORA_DIM; i++) j->V[r * ORA_DIM + i] = (int8_t)v[i];
        if (j->dot) j->dot[r] = d;
    }
    return NULL;
}

int ora_search_batch(ora_codec *c, int32_t m_max, int32_t mode, double scale, int64_t n,
                     const float *X, int8_t *V, double *dot, int32_t nthreads) {
    if (!c->store_all || m_max < 2 || m_max > c->M || n < 0) return -1;
    if (nthreads < 1) nthreads = 1;
    search_job *jobs = calloc((size_t)nthreads, sizeof(search_job));
    pthread_t *th = calloc((size_t)nthreads, sizeof(pthread_t));
    if (!jobs || !th) { free(jobs); free(th); return -2; }
    for (int t = 0; t < nthreads; t++) {
        search_job jb = {c, m_max, mode, t, nthreads, 0, scale, n, X, V, dot};
        jobs[t] = jb;
        pthread_create(&th[t], NULL, search_thread, &jobs[t]);
    }
    int bad = 0;
    for (int t = 0; t < nthreads; t++) { pthread_join(th[t], NULL); bad |= jobs[t].bad; }
    free(jobs); free(th);
    return bad ? -1 : 0;
}

/* ---- brute force: every point of shells 2..m_max from the congruences ----------------- */
typedef struct {
    int m_max, mode, target_sum8;
    double scale;
    int64_t n;
    const double *Y;            /* [n][24] */
    int res[ORA_DIM];           /* residue mod 4 each coordinate must have */
    int minrest[ORA_DIM + 1];   /* least squared norm coordinates i.. can take */
    int x[ORA_DIM];
    double *part;               /* [25][n]: <y, x> over the first i coordinates */
    double *best, *bestdot;     /* [n] */
    int32_t *bestv;             /* [n][24] */
    int64_t visited;
} brute_ctx;

static void brute_rec(brute_ctx *e, int i, int rem, int sum) {
    if (i == ORA_DIM) {
        int norm2 = 16 * e->m_max - rem;
        if (norm2 < 32 || mod_pos(sum, 8) != e->target_sum8) return;   /* shell >= 2, mod 8 */
        e->visited++;
        const double *d = e->part + (size_t)ORA_DIM * e->n;
        for (int64_t t = 0; t < e->n; t++) {
            double f = search_objective(e->mode, e->scale, d[t], norm2);
            if (f > e->best[t]) {
                e->best[t] = f;
                e->bestdot[t] = d[t];
                for (int k = 0; k < ORA_DIM; k++) e->bestv[t * ORA_DIM + k] = e->x[k];
            }
        }
        return;
    }
    int vmax = (int)floor(sqrt((double)rem)) + 1;
    for (int v = -vmax; v <= vmax; v++) {
        if (mod_pos(v, 4) != e->res[i]) continue;
        int r2 = rem - v * v;
        if (r2 < e->minrest[i + 1]) continue;
        e->x[i] = v;
        const double *p = e->part + (size_t)i * e->n;
        double *q = e->part + (size_t)(i + 1) * e->n;
        for (int64_t t = 0; t < e->n; t++) q[t] = p[t] + e->Y[t * ORA_DIM + i] * (double)v;
        brute_rec(e, i + 1, r2, sum + v);
    }
}

typedef struct {
    brute_ctx e;
    int tid, nthreads;
} brute_job;

static void *brute_thread(void *arg) {
    brute_job *j = arg;
    brute_ctx *e = &j->e;
    for (int job = j->tid; job < 2 * 4096; job += j->nthreads) {   /* (coset, codeword) */
        int odd = job / 4096;
        uint32_t cw = g_golay_mask[job % 4096];
        e->target_sum8 = odd ? 4 : 0;
        for (int i = 0; i < ORA_DIM; i++) {
            int in = (int)(cw >> i & 1u);
            e->res[i] = odd ? (in ? 1 : 3) : (in ? 2 : 0);
        }
        e->minrest[ORA_DIM] = 0;
        for (int i = ORA_DIM - 1; i >= 0; i--)
            e->minrest[i] = e->minrest[i + 1] + (e->res[i] == 0 ? 0 : (e->res[i] == 2 ? 4 : 1));
        brute_rec(e, 0, 16 * e->m_max, 0);
    }
    return NULL;
}

int64_t ora_search_brute(int32_t m_max, int32_t mode, double scale, int64_t n, const float *X,
                         int8_t *V, double *dot, int32_t nthreads) {
    if (m_max < 2 || (mode != 0 && mode != 1) || (mode == 1 && !(scale > 0.0)) || n < 0) return -1;
    ensure_golay();
    if (nthreads < 1) nthreads = 1;
    double *Y = malloc(sizeof(double) * (size_t)(n * ORA_DIM + 1));
    brute_job *jobs = calloc((size_t)nthreads, sizeof(brute_job));
    pthread_t *th = calloc((size_t)nthreads, sizeof(pthread_t));
    if (!Y || !jobs || !th) { free(Y); free(jobs); free(th); return -2; }
    for (int64_t k = 0; k < n * ORA_DIM; k++) Y[k] = (double)X[k];
    int ok = 1;
    for (int t = 0; t < nthreads; t++) {
        brute_ctx *e = &jobs[t].e;
        e->m_max = m_max; e->mode = mode; e->scale = scale; e->n = n; e->Y = Y;
        e->part = calloc((size_t)(ORA_DIM + 1) * (size_t)(n + 1), sizeof(double));
        e->best = malloc(sizeof(double) * (size_t)(n + 1));
        e->bestdot = calloc((size_t)(n + 1), sizeof(double));
        e->bestv = calloc((size_t)(n + 1) * ORA_DIM, sizeof(int32_t));
        if (!e->part || !e->best || !e->bestdot || !e->bestv) ok = 0;
        else for (int64_t k = 0; k < n; k++) e->best[k] = -INFINITY;
        jobs[t].tid = t;
        jobs[t].nthreads = nthreads;
    }
    int64_t visited = 0;
    if (ok) {
        for (int t = 0; t < nthreads; t++) pthread_create(&th[t], NULL, brute_thread, &jobs[t]);
        for (int t = 0; t < nthreads; t++) { pthread_join(th[t], NULL); visited += jobs[t].e.visited; }
        for (int64_t k = 0; k < n; k++) {          /* best over the threads */
            int bt = 0;
            for (int t = 1; t < nthreads; t++)
                if (jobs[t].e.best[k] > jobs[bt].e.best[k]) bt = t;
            for (int i = 0; i < ORA_DIM; i++) V[k * ORA_DIM + i] = (int8_t)jobs[bt].e.bestv[k * ORA_DIM + i];
            if (dot) dot[k] = jobs[bt].e.bestdot[k];
        }
    }
    for (int t = 0; t < nthreads; t++) {
        free(jobs[t].e.part); free(jobs[t].e.best); free(jobs[t].e.bestdot); free(jobs[t].e.bestv);
    }
    free(Y); free(jobs); free(th);
    return ok ? visited : -2;
}

/* The best point of one class and one codeword (the rearrangement rules above), exposed so
 * that tests can check them against an exact assignment solver.  word: the 1-mod-4 set T
 * (odd class, any codeword) or the 2-mod-4 set S (even class, a codeword of weight k).
 * Returns 0, or -1 when the class does not exist or the word does not fit it. */
int ora_class_best(ora_codec *c, int32_t m, int64_t j, uint32_t word, const double y[ORA_DIM],
                   int32_t v_out[ORA_DIM], double *dot_out) {
    if (m < 2 || m > c->M || build_shell(c, m) || j < 0 || j >= c->ncls[m]) return -1;
    const ocls *o = &c->cls[m][j];
    int ok = golay_contains(c->golay_mask, word & 0xFFFFFFu, NULL) && word <= 0xFFFFFFu &&
             (o->odd || popcount24(word) == o->k);
    if (ok) {
        int ord[ORA_DIM], v[ORA_DIM];
        order_desc(y, ord);
        if (o->odd) best_odd(o, word, y, ord, v); else best_even(o, word, y, ord, v);
        for (int i = 0; i < ORA_DIM; i++) v_out[i] = v[i];
        if (dot_out) *dot_out = dot24(y, v);
    }
    drop_shell(c, m);
    return ok ? 0 : -1;
}

/* ===================================================================================== */
/* Spherical GPTQ, one pass ([notes-K3] 关键设计 3 "保模长球面曲率反馈": the shape-gain        */
/* candidate is rescaled to the original norm, w^ = (|w| / |w~|) w~, a retraction onto the   */
/* product of spheres; the residual E = w - w^ is propagated to the unquantized weights      */
/* through U = chol(H^-1)^T).  Readings:                                                     */
/*   - blocks of 24 columns, in column order; each row's block is quantized jointly: its     */
/*     direction is the angular search over shells 2..max_shell of the block rounded to fp32 */
/*     (the search's input type), and w~ = g v / |v| for any gain g, so w^ = |w| v / |v|;     */
/*   - the propagation is the joint (block) form of GPTQ's update: with H^-1 = U^T U (U upper */
/*     triangular), the inverse Hessian of the columns not yet quantized is the trailing     */
/*     block of U^T U, so quantizing block B with error E moves the later columns by          */
/*     -E U_BB^-1 U_B,rest (one column at a time this is GPTQ's -e / U_ii * U_i,rest);        */
/*   - fixed operation order, so that another implementation can reproduce it bit for bit:    */
/*     |w|^2 = fma chain over i ascending; ratio = sqrt(|w|^2) / sqrt(16 m); w^_i = ratio v_i; */
/*     G_B = U_BB^-1 U_B,rest by back substitution per column (g_i = (u_i - sum_{k>i}          */
/*     U_ik g_k) / U_ii, the sum as an fma chain over k ascending from u_i); the update       */
/*     W[r][c] -= (fma chain over k ascending of E_k G_B[k][c], from 0).                      */
/* ===================================================================================== */

int ora_gptq_block_matrix(int32_t cols, const double *U, int32_t b, double *G) {
    /* G [24][cols]: G_B[k][c] for c >= 24 (b + 1), 0 elsewhere */
    if (cols % 24 || b < 0 || b >= cols / 24) return -1;
    const int base = 24 * b;
    for (int k = 0; k < 24; k++)
        for (int c = 0; c < cols; c++) G[(size_t)k * cols + c] = 0.0;
    for (int c = base + 24; c < cols; c++) {
        for (int i = 23; i >= 0; i--) {
            double acc = U[(size_t)(base + i) * cols + c];
            for (int k = i + 1; k < 24; k++)
                acc = fma(-U[(size_t)(base + i) * cols + base + k], G[(size_t)k * cols + c], acc);
            G[(size_t)i * cols + c] = acc / U[(size_t)(base + i) * cols + base + i];
        }
    }
    return 0;
}

int ora_spherical_gptq(ora_codec *c, int32_t max_shell, int32_t rows, int32_t cols, double *W, const double *U,
                       int8_t *points, double *norms) {
    if (!c->store_all || max_shell < 2 || max_shell > c->M || rows < 0 || cols <= 0 || cols % 24) return -1;
    const int nb = cols / 24;
    double *G = malloc(sizeof(double) * (size_t)24 * cols);
    double *E = malloc(sizeof(double) * 24 * (size_t)(rows > 0 ? rows : 1));
    if (!G || !E) { free(G); free(E); return -2; }
    int rc = 0;
    for (int b = 0; b < nb && rc == 0; b++) {
        ora_gptq_block_matrix(cols, U, b, G);
        for (int r = 0; r < rows; r++) {
            double *w = W + (size_t)r * cols + 24 * b;
            double y[ORA_DIM], s = 0.0, d;
            int32_t v[ORA_DIM];
            for (int i = 0; i < ORA_DIM; i++) y[i] = (double)(float)w[i];
            if (ora_search(c, max_shell, 0, 1.0, y, v, &d)) { rc = -1; break; }
            int n2 = 0;
            for (int i = 0; i < ORA_DIM; i++) { s = fma(w[i], w[i], s); n2 += v[i] * v[i]; }
            const double ratio = sqrt(s) / sqrt((double)n2);
            for (int i = 0; i < ORA_DIM; i++) {
                const double what = ratio * (double)v[i];
                E[(size_t)r * 24 + i] = w[i] - what;
                w[i] = what;
                points[((size_t)r * nb + b) * 24 + i] = (int8_t)v[i];
            }
            norms[(size_t)r * nb + b] = sqrt(s);
        }
        for (int r = 0; r < rows && rc == 0; r++)
            for (int col = 24 * (b + 1); col < cols; col++) {
                double acc = 0.0;
                for (int k = 0; k < 24; k++) acc = fma(E[(size_t)r * 24 + k], G[(size_t)k * cols + col], acc);
                W[(size_t)r * cols + col] -= acc;
            }
    }
    free(G);
    free(E);
    return rc;
}
