/*
 * llvq.h -- C ABI of libllvq: Leech lattice vector quantization (LLVQ) decode, encode and
 * fused decode-and-multiply on one NVIDIA B200 (sm_100a), for 48-, 72- and 96-bit block indices
 * (2, 3 and 4 bits per weight).
 *
 * What the calls compute ("Leech Lattice Vector Quantization for Efficient LLM Compression",
 * arXiv 2603.11021):
 *   - A packed word carries one block index I into the union of Leech lattice shells
 *     m = 2..M (shell m: squared norm 2m; papernotes.org notes, 方法详解 / 关键设计 1).
 *   - I decodes by the hierarchical bijection of 关键设计 2: the shell from cumulative shell
 *     offsets, the class (magnitude multiset + even/odd coset) from class offsets, then
 *     r = I_class mod A (Golay codeword), I' = floor(I_class / A), s = I' mod 2^B (signs),
 *     I'' = floor(I' / 2^B) (lexicographic arrangement rank).  The result is a 24-dim integer
 *     vector of the sqrt(8)-scaled Leech lattice (sum of squares 16 m).
 *   - The fused calls scale each block vector by its shape-gain gain and accumulate its dot
 *     product with fp16 activations, never writing dequantized weights to memory (关键设计 4;
 *     gist.science summary, Methodik 4 "Dequantisierungskernel").
 * The concrete index format (Golay generator, class order, sign order, arrangement order)
 * is fixed by the readings documented with the repository.
 *
 * Conventions for every call:
 *   - Pointers named d_* are DEVICE pointers on the device current when the codec was
 *     created; they are owned by the caller and must stay valid until the stream has run
 *     the call.  Host pointers are plain host memory.
 *   - `stream` is a cudaStream_t passed as void* (NULL = the legacy default stream).
 *   - Calls validate their arguments on the host and return LLVQ_ERR_ARG without launching
 *     anything when a check fails.  Launch failures return LLVQ_ERR_CUDA.  No call allocates
 *     device memory or synchronises, except llvq_codec_create/destroy and llvq_get_error.
 *   - Device-side faults in the data (an index >= N_M; for llvq_encode, a vector outside the
 *     coded set) do not trap: the block decodes to the zero vector (the vector encodes to an
 *     invalid index) and a sticky flag is set, read back by llvq_get_error.
 *   - Kernels are written for sm_100a only; there is no CPU fallback.
 */
#ifndef LLVQ_H
#define LLVQ_H
#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    LLVQ_OK = 0,
    LLVQ_ERR_ARG = 1,          /* invalid argument: null pointer, size, alignment, mismatch */
    LLVQ_ERR_UNSUPPORTED = 2,  /* valid request the library does not implement */
    LLVQ_ERR_CUDA = 3,         /* CUDA runtime error (no device, launch failure, ...) */
    LLVQ_ERR_DEVICE_FLAG = 4   /* a kernel raised a sticky data flag (see llvq_get_error) */
} llvq_status;

typedef enum {
    LLVQ_GAIN_FP16_DIRECT = 0, /* gains: fp16 [rows][blocks_per_row]; weight = g * v */
    LLVQ_GAIN_U8_TABLE = 1     /* gains: fp16 [rows][256], code in the word's 8 bits above the
                                  index; weight = table[code] * v / |v|, |v| = 4 sqrt(m)
                                  (shape-gain: unit direction times a scalar gain) */
} llvq_gain_mode;

/* Sticky device flags returned by llvq_get_error. */
#define LLVQ_FLAG_INDEX_RANGE 0x1u  /* some index was >= N_M (its block decoded to zero) */
#define LLVQ_FLAG_WAIT_TIMEOUT 0x2u /* a bounded wait (table copy, tensor-core products) gave up;
                                       the output of that call is incomplete */
#define LLVQ_FLAG_NOT_CODED 0x4u    /* llvq_encode met a vector that is not a coded lattice point */
#define LLVQ_FLAG_SEARCH_INPUT 0x8u /* llvq_search met a row holding a NaN or an infinity */

/* Criteria of llvq_search. */
#define LLVQ_SEARCH_ANGULAR 0       /* maximize <x, v> / |v| (the shape of a shape-gain split) */
#define LLVQ_SEARCH_EUCLIDEAN 1     /* minimize |x - scale * v| (spherical clipping) */

/* Opaque codec: owns the decode tables of one index budget on one device. */
typedef struct llvq_codec llvq_codec;

/* A compressed weight matrix W [rows][cols], split into 24-weight blocks along cols.
 * words: device, [rows][row_pitch_words] packed words of word_bytes bytes (row-major).
 *   word_bytes 8  (index_bits 48): bits [0,48) index, [48,56) gain code, [56,64) zero.
 *   word_bytes 16 (index_bits 72): little-endian; bits [0,72) index, [72,80) gain code.
 *   word_bytes 16 (index_bits 96): little-endian; bits [0,96) index, [96,104) gain code.
 * Block j of row r covers columns [24 j, 24 j + 24); cols beyond the logical width are
 * padding, and the activations must be zero there.  Alignment: words 8-byte (16-byte for
 * 16-byte words) aligned, gains 2-byte aligned. */
typedef struct {
    int32_t rows;              /* M */
    int32_t cols;              /* K (logical); blocks_per_row = ceil(K / 24) */
    int32_t blocks_per_row;    /* nb */
    int32_t index_bits;        /* 48, 72 or 96; must equal the codec's */
    int32_t word_bytes;        /* 8 for 48-bit, 16 for 72- and 96-bit */
    int32_t gain_mode;         /* llvq_gain_mode */
    int64_t row_pitch_words;   /* >= blocks_per_row */
    const void *words;         /* device */
    const void *gains;         /* device fp16 (see llvq_gain_mode) */
} llvq_weight;

/* Build the tables for an index budget (48 -> shells 2..13, 72 -> shells 2..53, 96 -> shells
 * 2..214) on the current device and upload them (the union of shells m = 2..M and the
 * shell / class offsets of papernotes.org notes, 关键设计 1 and 2).  *out is owned by the caller and released with
 * llvq_codec_destroy.  Thread-safe to use from several streams afterwards (the codec is
 * read-only except for its sticky flag word).
 * 48 and 72 bits: tables of 76 KB / 11 MB, built in well under a second.  96 bits: 304,649,365
 * class records of 64 bytes, a 1 GB guide and 2.4 GB of encoder class keys (about 23 GB of device
 * memory), built on all host cores and the device (several seconds; a few GB of host memory while
 * it runs); LLVQ_ERR_CUDA when the device memory is not available, with the reason in
 * llvq_last_error_message. */
llvq_status llvq_codec_create(int32_t index_bits, llvq_codec **out);
void llvq_codec_destroy(llvq_codec *codec);

/* Host query: largest shell M, number of coded points N_M (as lo/hi 64-bit halves) and the
 * number of classes (papernotes.org notes, 关键设计 1: the union's cumulative size N_M).  Any output
 * pointer may be NULL. */
llvq_status llvq_codec_info(const llvq_codec *codec, int32_t *max_shell, uint64_t *n_points_lo,
                            uint64_t *n_points_hi, int64_t *n_classes);

/* Decode n packed words (their index bits; gain bits are ignored) into int8 d_out [n][24]
 * (the lattice coordinates), by the hierarchical bijection of papernotes.org notes, 关键设计 2
 * (shell, class, then r = I_class mod A, s, I'' by div/mod).  d_words: device, n words of word_bytes (8 or 16, matching the
 * codec), aligned to word_bytes.  d_out: device, 24*n bytes, 8-byte aligned.  n >= 0. */
llvq_status llvq_decode(const llvq_codec *codec, const void *d_words, int32_t word_bytes, int64_t n,
                        int8_t *d_out, void *stream);

/* Encode n lattice points into packed words: the inverse of llvq_decode (the pages describe
 * the conversion to and from bitstrings; papernotes.org notes, 关键设计 2).  d_vectors: device
 * int8 [n][24] in the sqrt(8)-scaled coordinates llvq_decode produces, 8-byte aligned.  d_words:
 * device, n words of word_bytes (8 for the 48-bit budget, 16 for the 72- and 96-bit budgets),
 * aligned to word_bytes, written with the index in the index bits and a zero gain code.  A vector that is not a point of the coded shells (wrong coset
 * congruences, not a Golay codeword pattern, shell outside 2..M, the zero vector) gets the index
 * 2^index_bits - 1, which decodes to zero, and raises LLVQ_FLAG_NOT_CODED.  n >= 0. */
llvq_status llvq_encode(const llvq_codec *codec, const int8_t *d_vectors, int64_t n, void *d_words,
                        int32_t word_bytes, void *stream);

/* Fused decode-and-multiply, batch 1 (papernotes.org notes, 关键设计 4: the GPU fused dequantization
 * kernel; gist.science, Methodik 4): d_y[r] = sum_j scale(r, j) * <v(r, j), x[24 j .. 24 j + 23]>
 * with fp32 accumulation.  d_x: device fp16 [blocks_per_row * 24] (zero beyond cols), 16-byte
 * aligned.  d_y: device fp32 [rows], 4-byte aligned, overwritten. */
llvq_status llvq_gemv(const llvq_codec *codec, const llvq_weight *w, const void *d_x, float *d_y,
                      void *stream);

/* Fused decode-and-multiply for 1 <= batch <= 16 (papernotes.org notes, 关键设计 4; the batch-1
 * call above with a small batch of activations): d_Y[b][r] for activations d_X [batch][nb*24]
 * (fp16, row stride nb*24, zero beyond cols, 16-byte aligned).  Each block is decoded once for the
 * whole batch.  d_Y: device fp32 [batch][rows], overwritten.  48-bit batches of 8 or more run on
 * the tensor cores: decoded 128-row tiles (exact fp16 integers) times a block-diagonal activation
 * tile, per-block partial dots in TMEM, gains applied in fp32; that path zeroes d_Y on the stream
 * first and adds K-split partial sums atomically (summation order not fixed).  72/96-bit batches
 * run on the CUDA cores at every size (their decode dominates). */
llvq_status llvq_gemm_smallbatch(const llvq_codec *codec, const llvq_weight *w, const void *d_X,
                                 int32_t batch, float *d_Y, void *stream);

/* Decode without any device allocation.  Some callers cannot call cudaMalloc: a plug-in whose
 * device memory is all owned by a framework's caching allocator, or a latency-critical path
 * where cudaMalloc's implicit device synchronisation is not allowed.  They cannot create a codec
 * (llvq_codec_create allocates its tables), so this entry point keeps what the decode kernel
 * needs besides its input and output -- the 48-bit table image and a status word -- in one
 * static device array inside the library: 76,544 bytes on every device that loads the library,
 * held until the process exits.  The paper has no counterpart; this is a packaging variant of
 * llvq_decode for the 48-bit budget only (index_bits must be 48, word_bytes 8; anything else is
 * LLVQ_ERR_UNSUPPORTED / LLVQ_ERR_ARG).  It calls no cudaMalloc, cudaFree or allocating library
 * routine.  The first call on a device builds the tables on the host and copies them into the
 * array synchronously (set-up, once per device).  Do not reset the device after that call: the
 * library keeps the array's address and would not copy the tables again.  Calls share the
 * array, and calls that overlap on the GPU race on its status word.  An index >= N_M decodes to
 * the zero vector (a coded point is never zero); no call reports it -- llvq_get_error reads a
 * codec's flags, not this array -- so zero rows are the only sign of such an index.  Arguments
 * as for llvq_decode. */
llvq_status llvq_decode_noalloc(int32_t index_bits, const void *d_words, int32_t word_bytes, int64_t n,
                                int8_t *d_out, void *stream);

/* Host-side inspection of the 96-bit class table (no device needed): the class records of shell
 * m (2 <= m <= 214) in index order, as the decoder reads them.  A class is one multiset of |x_i|
 * in one coset; its magnitude groups form one list (even coset: the magnitudes 0 mod 4 ascending,
 * then those 2 mod 4 ascending; odd coset: all ascending).  Fields:
 *   start (start_lo, low 32 bits of start_hi): first global index of the class (< 2^96);
 *   meta: bits 0..6 t = bitlen(P - 1) (P = arrangements of the class), 7..14 shell m,
 *         15..19 k (even: codeword weight), 20..24 B (free sign bits), 25 odd coset,
 *         26 parity target (even: sum|x|/4 mod 2);
 *   rcp_lo/rcp_hi: ceil(2^(128 + t) / P) - 2^128;
 *   cum: byte g = 0x7F + (number of coordinates in groups 0..g), 16 groups (unused: 0x7F + 24);
 *   vals: byte g = magnitude of group g (unused: 0).
 * out may be NULL (then only *n_classes is set); otherwise it holds capacity records and the call
 * returns LLVQ_ERR_ARG when the shell has more.  The first call builds the shell sizes and class
 * counts (a few seconds on all host cores) and keeps them for later calls. */
typedef struct {
    uint64_t start_lo;
    uint32_t start_hi;
    uint32_t meta;
    uint64_t rcp_lo, rcp_hi;
    uint32_t cum[4];
    uint32_t vals[4];
} llvq_class96;
llvq_status llvq_class_table96(int32_t m, llvq_class96 *out, int64_t capacity, int64_t *n_classes);

/* Nearest-point search over the shell union Shell(2) u ... u Shell(max_shell) of the 48-bit
 * budget: for each row x of d_X, the lattice point v (sqrt(8)-scaled coordinates, |v|^2 = 16 m on
 * shell m) that maximizes <x, v> / |v| (LLVQ_SEARCH_ANGULAR: the direction of a shape-gain split)
 * or minimizes |x - scale * v| (LLVQ_SEARCH_EUCLIDEAN: spherical clipping, reconstruction
 * scale * v).  Source: papernotes.org notes, 方法详解 / 关键设计 1 (search over the union of shells,
 * unit vectors compared by their inner product for the shape-gain split) and gist.science,
 * Methodik 2 (Euclidean distance for spherical shaping, cosine similarity for shape-gain, both
 * over the union; an extension of Adoul & Barth's single-shell search).  The search is exact: it
 * takes the best point of every class and Golay codeword in closed form (rearrangement of the
 * sorted |x_i|), in fp64.  Ties between equally good points go to the lower class (index order),
 * then the lower codeword mask.
 *   codec: 48-bit (others: LLVQ_ERR_UNSUPPORTED); 2 <= max_shell <= 13.  Shells 2..11 fit 46
 *     index bits, 2..12 47 bits, 2..13 48 bits; every point found encodes with llvq_encode.
 *   scale: Euclidean only, finite and > 0 (ignored by the angular criterion).
 *   d_X: device fp32 [n][24], 4-byte aligned.  d_points: device int8 [n][24], overwritten.
 *   d_dots: device fp64 [n] (<x, v>), 8-byte aligned, or NULL.
 *   d_gain_levels / n_levels / d_gain_codes: angular only, optional (all NULL / 0, or all set with
 *     1 <= n_levels <= 256): d_gain_codes[i] = the level nearest to <x, v> / |v| (the best gain for
 *     the direction v / |v|), ties to the lower level; device fp64 levels, 8-byte aligned; device
 *     uint8 codes.
 * A row holding a NaN or an infinity gets the zero point, a NaN dot and code 0, and raises
 * LLVQ_FLAG_SEARCH_INPUT.  One CTA per row (one resident per SM); no allocation. */
llvq_status llvq_search(const llvq_codec *codec, int32_t max_shell, int32_t mode, double scale,
                        const float *d_X, int64_t n, int8_t *d_points, double *d_dots,
                        const double *d_gain_levels, int32_t n_levels, uint8_t *d_gain_codes,
                        void *stream);

/* One pass of Spherical GPTQ over a weight matrix W [rows][cols] on the 48-bit union
 * (papernotes.org notes, 方法详解 / 关键设计 3 "保模长球面曲率反馈": the shape-gain candidate w~ is
 * rescaled to the original norm, w^ = (|w| / |w~|) w~, a retraction onto the product of spheres,
 * and the residual E = w - w^ is propagated to the weights not yet quantized through
 * U = chol(H^-1)^T).  For each 24-column block B in column order: every row's block w gets its
 * direction v from the angular search over shells 2..max_shell (the block rounded to fp32), is
 * replaced by w^ = |w| v / |v| (so the gain drops out), and the later columns move by -E G_B with
 * G_B = U_BB^-1 U_B,rest (GPTQ's update in block form).  fp64 throughout, in a fixed operation
 * order (stated in csrc/gptq48.cuh) that makes the result reproducible bit for bit.
 *   codec: 48-bit (others: LLVQ_ERR_UNSUPPORTED); 2 <= max_shell <= 13.
 *   d_W: device fp64 [rows][cols], row-major, 8-byte aligned, overwritten: each block ends as
 *     its retraction; 0 <= rows <= 65535; cols > 0 a multiple of 24.  Finite values only (a
 *     non-finite row raises LLVQ_FLAG_SEARCH_INPUT and its results are unspecified).
 *   d_U: device fp64 [cols][cols], upper triangular with H^-1 = U^T U (the caller factors its
 *     calibration Hessian, e.g. with a library Cholesky); only the upper triangle is read.
 *   d_points: device int8 [rows][cols / 24][24]: v per block.  d_norms: device fp64
 *     [rows][cols / 24], 8-byte aligned: |w| per block when it was quantized (the gain a gain
 *     quantizer would code).
 *   d_workspace: device, 256-byte aligned, at least llvq_spherical_gptq_workspace(rows, cols)
 *     bytes (cols^2 x 8 for the block matrices, plus 36 bytes per row), owned by the caller.
 * Launches 1 + 4 (cols / 24) kernels on `stream`; no allocation. */
size_t llvq_spherical_gptq_workspace(int32_t rows, int32_t cols);
llvq_status llvq_spherical_gptq(const llvq_codec *codec, int32_t max_shell, int32_t rows, int32_t cols,
                                double *d_W, const double *d_U, int8_t *d_points, double *d_norms,
                                void *d_workspace, size_t workspace_bytes, void *stream);

/* Synchronise `stream`, return the sticky device flags raised since the last call in *flags
 * and clear them.  Returns LLVQ_ERR_DEVICE_FLAG when any flag was set, LLVQ_OK otherwise. */
llvq_status llvq_get_error(const llvq_codec *codec, void *stream, uint32_t *flags);

/* Static string for a status code. */
const char *llvq_status_string(llvq_status status);

/* The reason of the last failed call on this thread that gave one (table construction, device
 * memory), or an empty string.  Valid until the next call on this thread. */
const char *llvq_last_error_message(void);

/* Limits of the kernels' bounded waits, for tests of the timeout paths.  The paper has no
 * counterpart.  A kernel waits at most table_polls polls for its table copy into shared memory
 * and at most mma_polls polls for each round of its tensor-core products (tcgen05.mma completion);
 * when a wait gives up the kernel raises LLVQ_FLAG_WAIT_TIMEOUT (read by llvq_get_error), skips
 * the rest of its work (its outputs are then unspecified), and before it exits waits again, up to
 * the default limit, for the copy or the products in flight, so that nothing is still writing the
 * memory it releases.  0 makes the first wait give up at once; 0xFFFFFFFF restores the defaults
 * (2^22 and 2^20 polls).  Applies to launches made after the call, process-wide. */
void llvq_set_wait_polls(uint32_t table_polls, uint32_t mma_polls);

#ifdef __cplusplus
}
#endif
#endif /* LLVQ_H */
