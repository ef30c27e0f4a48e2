/*
 * llvq_oracle.h -- plain, slow, obviously-correct CPU oracle for LLVQ decode and GEMV.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may include, link or call this
 * code; only the tests, the package's smoke check and the bench's CPU-baseline leg use it.
 * It shares no code, header, table or constant with the CUDA library.
 *
 * Source of the method: "Leech Lattice Vector Quantization for Efficient LLM Compression"
 * (arXiv 2603.11021) as summarised on papernotes.org (section "方法详解", items 关键设计 1
 * and 2: the shell union and the hierarchical bijective index with
 * r = I_class mod A, I' = floor(I_class / A), s = I' mod 2^B, I'' = floor(I' / 2^B)),
 * on gist.science (section "Methodik", item 1 "Struktur des Leech-Gitters" and item 3
 * "Indexierungsschema") and the abstract on gptget.net ("conversion to and from bitstrings
 * without materializing the codebook").  Where the pages leave a detail open the oracle
 * takes the readings listed in the repository's design notes (generator polynomial, class
 * order, sign order, lexicographic arrangement order).
 *
 * The last sections add the nearest-point search over the shell union and one pass of
 * Spherical GPTQ (关键设计 1 and 3).
 *
 * Indices are up to 96 bits wide; at this interface they travel as (lo, hi) uint64 pairs.
 */
#ifndef LLVQ_ORACLE_H
#define LLVQ_ORACLE_H
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define ORA_DIM 24

/* ---- extended binary Golay code G24 ------------------------------------------------ */
/* All 4096 codewords as 24-bit masks (bit i = coordinate i), sorted by mask ascending. */
int ora_golay_by_mask(uint32_t out[4096]);
/* All 4096 codewords sorted by (weight, mask); base[w] = first slot of weight w (base[25] = 4096). */
int ora_golay_by_weight(uint32_t out[4096], int32_t base[26]);

/* ---- Leech lattice (sqrt(8)-scaled integer coordinates) ---------------------------- */
/* 1 if x lies in the scaled Leech lattice (mod-2 / mod-4 / mod-8 congruences), else 0. */
int ora_in_leech(const int32_t x[ORA_DIM]);
/* Explicit enumeration of shell m (sum x_i^2 = 16 m).  Writes up to cap points to out
 * (row-major [n][24]; out may be NULL to count only) and returns the number of points. */
uint64_t ora_shell_enumerate(int32_t m, int32_t *out, uint64_t cap);
/* Shell sizes N(m), m = 0..mmax, by a coordinate-wise dynamic programme over the
 * congruence conditions (independent of the class formula). */
int ora_shell_counts_dp(int32_t mmax, uint64_t *lo, uint64_t *hi);

/* ---- multiset arrangement ranking (lexicographic), exposed for brute-force pins ----- */
/* Rank / unrank sequences of length n over the multiset given by cnt[0..nv) (value j
 * appears cnt[j] times; value order = index order).  rank is (lo, hi). */
int ora_unrank_arrangement(int32_t nv, const int32_t *cnt, uint64_t lo, uint64_t hi, int32_t *seq);
int ora_rank_arrangement(int32_t nv, const int32_t *cnt, int32_t n, const int32_t *seq,
                         uint64_t *lo, uint64_t *hi);

/* ---- the codec: shells m = 2..M, classes, bijection ------------------------------- */
typedef struct ora_codec ora_codec;

typedef struct {
    int32_t m;            /* shell */
    int32_t odd;          /* 0 = even coset, 1 = odd coset */
    int32_t k;            /* even: number of coordinates with |x| = 2 mod 4; odd: 0 */
    int32_t nvals;        /* number of distinct magnitudes */
    int32_t vals[ORA_DIM];/* distinct magnitudes, ascending */
    int32_t cnts[ORA_DIM];/* their multiplicities */
    uint32_t A;           /* number of Golay refinements r */
    int32_t B;            /* number of free sign bits */
    uint64_t P_lo, P_hi;  /* number of admissible arrangements of the magnitudes */
    uint64_t size_lo, size_hi;     /* A * 2^B * P */
    uint64_t offset_lo, offset_hi; /* first global index of the class */
} ora_class_info;

/* index_bits in {48, 72, 96}: M = largest shell with N_2 + ... + N_M <= 2^index_bits.
 * (96 bits builds shell totals only; per-shell class lists are built on demand.) */
ora_codec *ora_codec_create(int32_t index_bits);
void ora_codec_destroy(ora_codec *c);
int32_t ora_codec_max_shell(const ora_codec *c);
void ora_codec_npoints(const ora_codec *c, uint64_t *lo, uint64_t *hi);
/* Shell m's first global index (m in 2..M+1; m = M+1 gives N_M). */
void ora_codec_shell_offset(const ora_codec *c, int32_t m, uint64_t *lo, uint64_t *hi);
/* Number of classes of shell m (builds the shell's list if needed). */
int64_t ora_codec_shell_nclasses(ora_codec *c, int32_t m);
/* Class j of shell m (0-based within the shell). */
int ora_codec_shell_class(ora_codec *c, int32_t m, int64_t j, ora_class_info *out);

/* decode: index -> lattice vector.  Returns 0 on success, -1 if index >= N_M. */
int ora_decode(ora_codec *c, uint64_t lo, uint64_t hi, int32_t x[ORA_DIM]);
/* encode: lattice vector -> index.  Returns 0, or -1 if x is not a coded point. */
int ora_encode(ora_codec *c, const int32_t x[ORA_DIM], uint64_t *lo, uint64_t *hi);
/* Batch decode of indices given as (lo, hi) arrays into int8 [n][24]; returns the
 * number of out-of-range indices (their rows are written as zero). */
int64_t ora_decode_batch(ora_codec *c, int64_t n, const uint64_t *lo, const uint64_t *hi,
                         int8_t *out);
/* Batch decode returning the shell of each index as well (m = 0 for out-of-range). */
int64_t ora_decode_batch_shell(ora_codec *c, int64_t n, const uint64_t *lo, const uint64_t *hi,
                               int8_t *out, int32_t *shell);

/* ---- fp64 GEMV / small-batch GEMM on packed words ------------------------------------
 * words: [rows][row_pitch_words] packed words of word_bytes (8 or 16) bytes.  A word holds
 * the index in its low index_bits bits and an 8-bit gain code in the next 8 bits.
 * gain_mode 0 (direct): gains = fp16 bits [rows][nb]; weight = g * v.
 * gain_mode 1 (table) : gains = fp16 bits [rows][256]; weight = t[code] * v / |v|,
 *                       |v| = 4 sqrt(m) (shape-gain: unit direction times gain).
 * x: fp16 bits [batch][nb*24]; y: double [batch][rows].
 * y[b][r] = sum_j sum_t weight(r, j, t) * x[b][24 j + t], every term in fp64.
 * Returns the number of out-of-range indices met (their blocks contribute zero). */
int64_t ora_gemm(ora_codec *c, int32_t rows, int32_t nb, const void *words, int32_t word_bytes,
                 int64_t row_pitch_words, int32_t gain_mode, const uint16_t *gains,
                 const uint16_t *x, int32_t batch, double *y);
/* Same, with the rows split over nthreads host threads (used for the CPU baseline timing). */
int64_t ora_gemm_mt(const ora_codec *c, int32_t rows, int32_t nb, const void *words,
                    int32_t word_bytes, int64_t row_pitch_words, int32_t gain_mode,
                    const uint16_t *gains, const uint16_t *x, int32_t batch, double *y,
                    int32_t nthreads);
/* Exhaustive self-check of shells m_lo..m_hi (48/72-bit codecs): direct enumeration,
 * encode, one hit per index, decode round trip.  See the definition for result[]. */
int ora_check_shells(ora_codec *c, int32_t m_lo, int32_t m_hi, int32_t nthreads, int64_t result[7]);
/* ---- nearest-point search over the shell union Shell(2) u ... u Shell(m_max) ------------
 * mode 0 (angular, the shape of a shape-gain split): maximize <y, v> / |v|.
 * mode 1 (Euclidean, spherical clipping): minimize |y - scale * v|^2 (scale > 0).
 * v is in sqrt(8)-scaled integer coordinates; m_max <= the codec's largest shell.  The
 * search takes the best point of every class and Golay codeword (rearrangement rules in the
 * definition).  ora_search returns 0, or -1 on bad arguments; *dot_out = <y, v>. */
int ora_search(ora_codec *c, int32_t m_max, int32_t mode, double scale, const double y[ORA_DIM],
               int32_t v_out[ORA_DIM], double *dot_out);
/* The same over rows of X (fp32 [n][24], read as exact doubles), rows split over host threads;
 * V: int8 [n][24]; dot: [n] or NULL.  48/72-bit codecs only.  Returns 0, or -1. */
int ora_search_batch(ora_codec *c, int32_t m_max, int32_t mode, double scale, int64_t n,
                     const float *X, int8_t *V, double *dot, int32_t nthreads);
/* The best point (largest <y, v>) of class j of shell m among the points whose 1-mod-4 set
 * (odd class) or 2-mod-4 set (even class) is the codeword word.  Returns 0, or -1. */
int ora_class_best(ora_codec *c, int32_t m, int64_t j, uint32_t word, const double y[ORA_DIM],
                   int32_t v_out[ORA_DIM], double *dot_out);
/* Brute force over every point of shells 2..m_max, enumerated from the congruences alone
 * (no classes, no rearrangement).  Returns the number of points visited, or a negative
 * value on bad arguments. */
int64_t ora_search_brute(int32_t m_max, int32_t mode, double scale, int64_t n, const float *X,
                         int8_t *V, double *dot, int32_t nthreads);
/* ---- Spherical GPTQ, one pass (papernotes 关键设计 3) ----------------------------------
 * W: fp64 [rows][cols], cols = 24 nb, updated in place (each block ends as its retraction
 * |w| v / |v|).  U: fp64 [cols][cols], upper triangular with H^-1 = U^T U.  points: int8
 * [rows][nb][24] (the angular search's v per block); norms: [rows][nb] (|w| when quantized).
 * Operation order as stated in the definition.  Returns 0, or a negative value. */
int ora_spherical_gptq(ora_codec *c, int32_t max_shell, int32_t rows, int32_t cols, double *W, const double *U,
                       int8_t *points, double *norms);
/* G_B = U_BB^-1 U_B,rest of block b by back substitution, as [24][cols] (zero before the later
 * columns).  Returns 0, or -1 on bad arguments. */
int ora_gptq_block_matrix(int32_t cols, const double *U, int32_t b, double *G);
/* fp16 bits -> double (exact). */
double ora_half_to_double(uint16_t h);

#ifdef __cplusplus
}
#endif
#endif
