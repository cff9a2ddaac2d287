// Engram n-gram hash and embedding-table row gather (sm_100a).
//
// engram_hash on the page "DeepSeek 开源 TileKernels" (zhichai.net/topic/177618722),
// section "5. Engram — 条件记忆门控": the token ids of each token's trailing
// n-gram are mixed with multiplications and XOR into one 64-bit hash per
// n-gram layer, which is mapped to one row index in each of the layer's
// embedding tables; the rows are then gathered.
//
//     h          = XOR_i u64(tok[s - i]) * m[l][i]         (wrapping u64)
//     idx[l][j]  = h mod P[l][j]                           (unsigned)
//     rows[l][j] = table(l, j)[idx[l][j], 0:D]
//
// Work decomposition: one group of 8 lanes per (token, layer).  Every lane of
// the group computes the hash (2-3 multiplies), lane j of the group reduces it
// modulo P[l][j] (and P[l][j+8]) and writes that index, and the indices are
// passed around the group with shuffles.  The group then copies the J rows:
// lane c moves the 16-byte chunks c, c+8, ... of every row, with the loads of
// up to 8 rows issued before their stores so that each lane keeps 8 random
// row reads in flight.  Rows are read through the non-coherent path (hot rows
// of skewed id distributions hit in L1/L2) and written with streaming stores.
//
// The remainder uses a precomputed reciprocal: with inv = floor((2^64-1)/P),
// q = umulhi(h, inv) is floor(h/P) or one less, so r = h - q*P lies in [0, 2P)
// and one conditional subtraction gives exactly h mod P, for every P >= 1.
#pragma once

#include "common.cuh"

namespace engram {

constexpr int kHashMaxL = 4;        // n-gram layers
constexpr int kHashMaxN = 8;        // n-gram order
constexpr int kHashMaxJ = 16;       // tables per layer
constexpr int kHashMaxTables = kHashMaxL * kHashMaxJ;
constexpr int kHashThreads = 256;

struct HashParams {
    int64_t B, S;
    int64_t pad_id;
    int32_t L, J, D;                         // D: row width in bf16 values
    int32_t ngram_n[kHashMaxL];
    uint64_t mult[kHashMaxL][kHashMaxN];
    uint64_t P[kHashMaxTables];              // rows of table q = l*J + j
    uint64_t inv[kHashMaxTables];            // floor((2^64 - 1) / P[q])
    int64_t row0[kHashMaxTables];            // first row of table q in `tables`
    uint64_t inv_L, inv_S;                   // floor((2^64 - 1) / L), floor((2^64 - 1) / S)
};

__device__ __forceinline__ uint64_t mod_by_inverse(uint64_t h, uint64_t P, uint64_t inv)
{
    const uint64_t q = __umul64hi(h, inv);
    const uint64_t r = h - q * P;
    return r >= P ? r - P : r;
}

// Quotient and remainder of x by d >= 1 with the same reciprocal (the integer
// divisions the kernel needs by the runtime L and S, without a 64-bit divide).
__device__ __forceinline__ uint64_t div_by_inverse(uint64_t x, uint64_t d, uint64_t inv, uint64_t &rem)
{
    uint64_t q = __umul64hi(x, inv);
    uint64_t r = x - q * d;
    if (r >= d) {
        ++q;
        r -= d;
    }
    rem = r;
    return q;
}

// CPL: 16-byte chunks per lane per row (rows of up to 64 * CPL bf16 values).
template <int CPL>
__global__ void __launch_bounds__(kHashThreads)
hash_gather_kernel(const int64_t *__restrict__ tokens, const uint4 *__restrict__ tables,
                   int64_t *__restrict__ idx_out, uint4 *__restrict__ rows_out,
                   const __grid_constant__ HashParams p)
{
    const int lane = threadIdx.x & 31;
    const int gl = lane & 7;        // lane within the group
    const int gbase = lane & ~7;    // first lane of the group
    const int64_t T = p.B * p.S;
    const int64_t ngroups = T * p.L;
    const int chunks = p.D >> 3;
    const int64_t nwarps = (int64_t)gridDim.x * (blockDim.x >> 5);

    for (int64_t wid = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; wid * 4 < ngroups;
         wid += nwarps) {
        const int64_t gid = wid * 4 + (lane >> 3);
        const bool active = gid < ngroups;
        int l = 0;
        uint64_t h = 0;
        if (active) {
            uint64_t lr, sr;
            const int64_t t = (int64_t)div_by_inverse((uint64_t)gid, (uint64_t)p.L, p.inv_L, lr);
            l = (int)lr;
            div_by_inverse((uint64_t)t, (uint64_t)p.S, p.inv_S, sr);
            const int64_t s = (int64_t)sr;
            for (int i = 0; i < p.ngram_n[l]; ++i) {
                const int64_t tok = (s - i >= 0) ? __ldg(tokens + (t - i)) : p.pad_id;
                h ^= (uint64_t)tok * p.mult[l][i];
            }
        }
        const int q0 = l * p.J;
        int64_t my0 = 0, my1 = 0;   // this lane's indices: tables j = gl and j = gl + 8
        if (active && gl < p.J) {
            my0 = (int64_t)mod_by_inverse(h, p.P[q0 + gl], p.inv[q0 + gl]);
            if (idx_out != nullptr)
                __stcs(reinterpret_cast<long long *>(idx_out) + gid * p.J + gl, (long long)my0);
        }
        if (active && gl + 8 < p.J) {
            my1 = (int64_t)mod_by_inverse(h, p.P[q0 + gl + 8], p.inv[q0 + gl + 8]);
            if (idx_out != nullptr)
                __stcs(reinterpret_cast<long long *>(idx_out) + gid * p.J + gl + 8, (long long)my1);
        }
        if (rows_out == nullptr) continue;

        for (int jb = 0; jb < p.J; jb += 8) {   // warp-uniform
            const int64_t mine = (jb == 0) ? my0 : my1;
            uint4 buf[8][CPL];
#pragma unroll
            for (int jj = 0; jj < 8; ++jj) {
                const int64_t r = __shfl_sync(0xffffffffu, mine, gbase + jj);
                const int j = jb + jj;
                if (active && j < p.J) {
                    const uint4 *src = tables + (p.row0[q0 + j] + r) * chunks;
#pragma unroll
                    for (int c = 0; c < CPL; ++c) {
                        const int ch = gl + 8 * c;
                        if (ch < chunks) buf[jj][c] = __ldg(src + ch);
                    }
                }
            }
#pragma unroll
            for (int jj = 0; jj < 8; ++jj) {
                const int j = jb + jj;
                if (active && j < p.J) {
                    uint4 *dst = rows_out + (gid * p.J + j) * chunks;
#pragma unroll
                    for (int c = 0; c < CPL; ++c) {
                        const int ch = gl + 8 * c;
                        if (ch < chunks) __stcs(dst + ch, buf[jj][c]);
                    }
                }
            }
        }
    }
}

}  // namespace engram
