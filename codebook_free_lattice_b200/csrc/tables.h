// tables.h -- host-side construction of the LLVQ decode tables for the CUDA library.
//
// Builds, from first principles, the index-format tables the kernels read: the extended
// binary Golay code in two orders, the classes of every shell m = 2..M with their offsets,
// and the per-class constants of the decode.  Method: "Leech Lattice Vector Quantization for
// Efficient LLM Compression", papernotes.org notes, 方法详解 / 关键设计 2 (shell by cumulative
// offsets, classes = magnitude multiset + even/odd coset in contiguous ranges, digits
// r = I_class mod A, s = I' mod 2^B, I'' = lexicographic arrangement rank; an even class ranks
// its codeword positions and the other positions separately, I'' = p_S + P_S p_C).
#pragma once
#include <stdint.h>

#include <string>
#include <vector>

namespace llvq {

using u128 = unsigned __int128;

struct HostClass {
    int m = 0;                 // shell (sum of squares 16 m)
    bool odd = false;          // coset
    int k = 0;                 // even: number of coordinates with |x| = 2 (mod 4)
    // magnitude groups in decode order: even -> the 2-mod-4 magnitudes ascending, then the
    // 0-mod-4 magnitudes ascending; odd -> all magnitudes ascending
    std::vector<int> vals, cnts;
    int n_side0 = 0;           // groups on the codeword side (even: 2-mod-4 groups; odd: all)
    uint32_t A = 0;            // Golay refinements
    int B = 0;                 // free sign bits
    u128 P = 0;                // admissible arrangements, P_S * P_C
    u128 P_S = 1, P_C = 1;     // even: arrangements on S / on its complement; odd: P, 1
    u128 size = 0, start = 0;  // A * 2^B * P and first global index
    int sum_abs = 0;           // sum of magnitudes
};

struct HostTables {
    int index_bits = 0;
    int M = 0;                           // largest shell
    u128 n_points = 0;                   // N_M
    std::vector<u128> shell_start;       // shell_start[m], m = 2..M+1
    std::vector<HostClass> classes;      // global order
    uint32_t golay_by_mask[4096];        // codewords, ascending mask
    uint32_t golay_by_weight[4096];      // codewords, ascending (weight, mask)
    int weight_base[25];                 // first by-weight slot of each weight
};

// The 4096 codewords of the extended binary Golay code (24-bit masks), in message order.
void golay_code(uint32_t words[4096]);

// index_bits 48 or 72.  Returns false and sets err on failure.
bool build_host_tables(int index_bits, HostTables &out, std::string &err);

}  // namespace llvq
