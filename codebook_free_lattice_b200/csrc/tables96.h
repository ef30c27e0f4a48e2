// tables96.h -- host construction of the class table of the 96-bit index budget (4 bits per
// weight: shells 2..214, about 2.5 x 10^8 classes).
//
// "Leech Lattice Vector Quantization for Efficient LLM Compression", papernotes.org notes,
// 方法详解 / 关键设计 2: the shell of an index comes from cumulative shell offsets, the class
// from contiguous class ranges inside the shell, then r, s and the arrangement rank.  At this
// budget the classes are too many for shared memory, so every class becomes one 64-byte record
// in global memory (about 16 GB on the device); a guide on the top 28 index bits narrows the
// search to a few records.
//
// The records are built shell by shell, and shells are independent once their sizes are known,
// so the build runs on all host cores.  Shell sizes come from the theta series of the Leech
// lattice, N_m = 65520 / 691 (sigma_11(m) - tau(m)); the class sizes of every shell must add
// up to it (a self-check of the enumeration).
#pragma once
#include <stdint.h>

#include <string>
#include <vector>

namespace llvq {

using u128 = unsigned __int128;

// One class as the 96-bit decoder reads it.  Magnitude groups form one list: the groups off
// the codeword first (even coset: magnitudes 0 mod 4, ascending), then the groups on it
// (2 mod 4, ascending); an odd class has one list of all its magnitudes, ascending.
struct alignas(16) Rec96 {
    uint64_t start_lo;        // first global index of the class, bits 0..63
    uint32_t start_hi;        // bits 64..95
    uint32_t meta;            // t | m << 7 | k << 15 | B << 20 | odd << 25 | parity << 26
    uint64_t rcp_lo, rcp_hi;  // R' = ceil(2^(128 + t) / P) - 2^128, t = bitlen(P - 1)
    uint32_t cum[4];          // byte g: 0x7F + C_<=g (groups 0..15; unused groups hold 24)
    uint32_t vals[4];         // byte g: magnitude of group g
};
static_assert(sizeof(Rec96) == 64, "Rec96 layout");

constexpr int kRec96Groups = 16;
constexpr uint32_t kMeta96Odd = 1u << 25, kMeta96Parity = 1u << 26;
inline int meta96_t(uint32_t m) { return (int)(m & 0x7Fu); }
inline int meta96_m(uint32_t m) { return (int)((m >> 7) & 0xFFu); }
inline int meta96_k(uint32_t m) { return (int)((m >> 15) & 0x1Fu); }
inline int meta96_B(uint32_t m) { return (int)((m >> 20) & 0x1Fu); }

struct Tables96 {
    int M = 0;                             // largest shell with N_2 + ... + N_M <= 2^96
    u128 n_points = 0;                     // N_M
    std::vector<u128> shell_start;         // [m], m = 0..M+1 (first global index of shell m)
    std::vector<int64_t> shell_classes;    // [m]: classes in shell m
    std::vector<int64_t> shell_even;       // [m]: even-coset classes in shell m (they come first)
    std::vector<int64_t> class_base;       // [m]: global index of the first class of shell m
    int64_t n_classes = 0;
    uint32_t golay_by_mask[4096];          // codewords, ascending mask
    uint32_t golay_by_weight[4096];        // codewords, ascending (weight, mask)
    int weight_base[25];                   // first by-weight slot of each weight
    int words_of_weight[25];
};

// Shell sizes, M, the Golay tables and the number of classes of every shell (counted on
// `threads` host threads).  Returns false and sets err on failure.
bool build_tables96(Tables96 &T, int threads, std::string &err);

// The records of shell m (T.shell_classes[m] of them) into out, in index order.  Returns false
// and sets err when the class sizes do not add up to the shell size.
bool fill_shell96(const Tables96 &T, int m, Rec96 *out, std::string &err);

}  // namespace llvq
