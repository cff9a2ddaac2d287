// Engram gather backward (sm_100a): the transpose of the table-row gather.
//
// The Engram section of the page "DeepSeek 开源 TileKernels" (zhichai.net/topic/177618722,
// "5. Engram — 条件记忆门控") hashes each token's n-grams to one row of each
// embedding table and gathers those rows.  Training the tables needs the
// transpose of that gather: the gradient of every gathered row is added to the
// table row it was read from, so a row read by several tokens receives the sum
// of their gradients:
//
//     d_tables[row0(q) + idx[t][q]] += d_rows[t][q]      for every (t, q)
//
// Deterministic segmented reduction by sorting:
//   1. keys: entry e = t * LJ + q gets the key row0(q) + idx[e], its global row
//      (an index outside its table gets the key R, the row count, which sorts
//      last and is never written; the kernel records
//      ENGRAM_DEVICE_ERR_INDEX_RANGE instead of trapping);
//   2. a stable least-significant-digit radix sort of (key, e), 8 bits per
//      pass: a per-tile digit histogram, one exclusive scan over
//      [digit][tile], and a scatter whose within-tile ranks come from
//      __match_any_sync (stable: entries keep their position order);
//   3. the sorted entries are cut into fixed chunks of kSegChunk, one warp per
//      chunk.  Each run of equal keys (a segment: all the gradients of one
//      table row, in position order) is summed in fp64; a segment that lies
//      inside one chunk is added to d_tables at once, a segment that crosses
//      chunk boundaries leaves one fp64 partial per chunk (carry_b for the
//      piece that continues into the next chunk, carry_a for the last piece),
//      and a second kernel adds those partials in chunk order.
// Every sum has a fixed order, so the result is bitwise reproducible.  bf16
// gradients enter the fp64 sums exactly; the row's fp32 value is updated with
// one rounding: d_tables[r] = fp32((double)d_tables[r] + sum).
#pragma once

#include "common.cuh"
#include "hash_gather.cuh"

namespace engram {

constexpr unsigned kErrIndexRange = 2u;   // ENGRAM_DEVICE_ERR_INDEX_RANGE

constexpr int kSortThreads = 256;
constexpr int kSortWarps = kSortThreads / 32;
constexpr int kSortRounds = 16;
constexpr int kSortTile = kSortThreads * kSortRounds;   // entries per CTA tile
constexpr int kRadixBins = 256;
constexpr int kScanThreads = 1024;
constexpr int kSegChunk = 64;                           // sorted entries per warp
constexpr int kSegThreads = 256;
static_assert(kSortThreads == kRadixBins, "one thread per digit in the histogram epilogue");

struct GatherBwdParams {
    int64_t N;                          // entries: T * L * J
    int32_t LJ;                         // tables
    int32_t D;                          // row width in bf16 values (even)
    uint32_t R;                         // rows of all tables; the key of an invalid entry
    uint32_t P[kHashMaxTables];         // rows of table q
    uint32_t row0[kHashMaxTables];      // first global row of table q
};

// Global row of entry e, or p.R when its index lies outside its table.
__device__ __forceinline__ uint32_t gbwd_key(const int64_t *__restrict__ idx, int64_t e,
                                             const GatherBwdParams &p, bool record)
{
    const int q = (int)((uint32_t)e % (uint32_t)p.LJ);
    const int64_t r = __ldg(idx + e);
    if (r < 0 || r >= (int64_t)p.P[q]) {
        if (record) record_device_error(kErrIndexRange);
        return p.R;
    }
    return p.row0[q] + (uint32_t)r;
}

// ------------------------------------------------------------ radix sort ----

// Digit histogram of one tile: hist[digit * ntiles + tile].
template <bool FROM_IDX>
__global__ void __launch_bounds__(kSortThreads)
gbwd_hist_kernel(const int64_t *__restrict__ idx, const uint32_t *__restrict__ keys,
                 const __grid_constant__ GatherBwdParams p, int shift, uint32_t *__restrict__ hist)
{
    __shared__ uint32_t sh[kRadixBins];
    const int tid = threadIdx.x;
    sh[tid] = 0;
    __syncthreads();
    const int64_t base = (int64_t)blockIdx.x * kSortTile;
#pragma unroll 4
    for (int r = 0; r < kSortRounds; ++r) {
        const int64_t e = base + r * kSortThreads + tid;
        if (e < p.N) {
            const uint32_t key = FROM_IDX ? gbwd_key(idx, e, p, true) : keys[e];
            atomicAdd(&sh[(key >> shift) & 0xffu], 1u);
        }
    }
    __syncthreads();
    hist[(int64_t)tid * gridDim.x + blockIdx.x] = sh[tid];
}

// Exclusive prefix sum of hist[0, n) in place, one CTA.  n is a multiple of
// kRadixBins; each thread owns a contiguous range of a multiple of 4 entries.
__global__ void __launch_bounds__(kScanThreads)
gbwd_scan_kernel(uint32_t *__restrict__ hist, int64_t n)
{
    __shared__ uint32_t warp_excl[32];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t per = (((n + kScanThreads - 1) / kScanThreads) + 3) & ~int64_t(3);
    const int64_t lo = min(n, (int64_t)tid * per), hi = min(n, lo + per);
    uint4 *h4 = reinterpret_cast<uint4 *>(hist);
    uint32_t own = 0;
#pragma unroll 4
    for (int64_t i = lo; i < hi; i += 4) {
        const uint4 c = h4[i >> 2];
        own += c.x + c.y + c.z + c.w;
    }
    uint32_t inc = own;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t t = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += t;
    }
    if (lane == 31) warp_excl[warp] = inc;
    __syncthreads();
    if (warp == 0) {
        const uint32_t w = warp_excl[lane];
        uint32_t winc = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t t = __shfl_up_sync(0xffffffffu, winc, o);
            if (lane >= o) winc += t;
        }
        warp_excl[lane] = winc - w;
    }
    __syncthreads();
    uint32_t run = warp_excl[warp] + inc - own;
    for (int64_t i = lo; i < hi; i += 4) {
        uint4 c = h4[i >> 2];
        const uint4 in = c;
        c.x = run;
        c.y = run + in.x;
        c.z = c.y + in.y;
        c.w = c.z + in.z;
        run = c.w + in.w;
        h4[i >> 2] = c;
    }
}

// Stable scatter of one tile by the digit at `shift`.  Round r handles
// entries base + r * kSortThreads + tid, so (round, warp, lane) is position
// order.  Within a warp the rank among equal digits comes from
// __match_any_sync; across the warps of a round, from per-warp digit counts
// tagged with the round (no clearing between rounds); across rounds, from the
// running digit offsets in run[].
template <bool FROM_IDX>
__global__ void __launch_bounds__(kSortThreads)
gbwd_scatter_kernel(const int64_t *__restrict__ idx, const uint32_t *__restrict__ keys_in,
                    const uint32_t *__restrict__ vals_in, const __grid_constant__ GatherBwdParams p,
                    int shift, const uint32_t *__restrict__ hist, uint32_t *__restrict__ keys_out,
                    uint32_t *__restrict__ vals_out)
{
    __shared__ uint32_t run[kRadixBins];
    __shared__ uint32_t wcnt[kSortWarps][kRadixBins];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    run[tid] = hist[(int64_t)tid * gridDim.x + blockIdx.x];
    for (int i = tid; i < kSortWarps * kRadixBins; i += kSortThreads) (&wcnt[0][0])[i] = 0u;
    __syncthreads();
    const uint32_t below = (1u << lane) - 1u;
    const int64_t base = (int64_t)blockIdx.x * kSortTile;
    for (int r = 0; r < kSortRounds; ++r) {
        const int64_t e = base + r * kSortThreads + tid;
        const bool valid = e < p.N;
        uint32_t key = 0, val = 0;
        if (valid) {
            if (FROM_IDX) {
                key = gbwd_key(idx, e, p, false);
                val = (uint32_t)e;
            } else {
                key = keys_in[e];
                val = vals_in[e];
            }
        }
        const uint32_t d = valid ? (key >> shift) & 0xffu : (uint32_t)kRadixBins;
        const uint32_t peers = __match_any_sync(0xffffffffu, d);
        const bool leader = (__ffs(peers) - 1) == lane;
        const uint32_t tag = (uint32_t)(r + 1) << 8;
        if (valid && leader) wcnt[warp][d] = tag | (uint32_t)__popc(peers);
        __syncthreads();
        if (valid) {
            uint32_t pos = run[d] + (uint32_t)__popc(peers & below);
            for (int w = 0; w < warp; ++w) {
                const uint32_t c = wcnt[w][d];
                if ((c & ~0xffu) == tag) pos += c & 0xffu;
            }
            // pos < N whenever the histogram counted the same keys; the check
            // only keeps a caller that changed idx in between inside the buffers
            if (pos < (uint64_t)p.N) {
                keys_out[pos] = key;
                vals_out[pos] = val;
            } else {
                record_device_error(kErrIndexRange);
            }
        }
        __syncthreads();
        if (valid && leader) atomicAdd(&run[d], (uint32_t)__popc(peers));
    }
}

// ------------------------------------------------- segmented reduction ----

__device__ __forceinline__ uint32_t lane_key(uint32_t k0, uint32_t k1, int e)
{
    return __shfl_sync(0xffffffffu, e < 32 ? k0 : k1, e & 31);
}

// One warp per chunk of kSegChunk sorted entries.  Lane l owns the bf16
// column pairs l, l + 32, ... (PPL of them) of a row.  BATCH rows of d_rows
// (and the d_tables rows of the segments that complete in the batch) are
// loaded before they are used, so each warp keeps BATCH random row reads in
// flight.
template <int PPL>
__global__ void __launch_bounds__(kSegThreads)
gbwd_segment_kernel(const uint32_t *__restrict__ keys, const uint32_t *__restrict__ vals,
                    const __nv_bfloat162 *__restrict__ d_rows,
                    const __grid_constant__ GatherBwdParams p, float2 *__restrict__ d_tables,
                    double2 *__restrict__ carry_a, double2 *__restrict__ carry_b)
{
    constexpr int BATCH = 8 / PPL;
    constexpr uint32_t kNone = 0xffffffffu;   // never a key: keys are <= R < 2^32 - 1
    const int lane = threadIdx.x & 31;
    const int npairs = p.D >> 1;
    const int64_t nchunks = (p.N + kSegChunk - 1) / kSegChunk;
    const int64_t nwarps = (int64_t)gridDim.x * (kSegThreads / 32);
    for (int64_t c = ((int64_t)blockIdx.x * kSegThreads + threadIdx.x) >> 5; c < nchunks;
         c += nwarps) {
        const int64_t lo = c * kSegChunk;
        const int n = (int)min((int64_t)kSegChunk, p.N - lo);
        const uint32_t k0 = lane < n ? keys[lo + lane] : kNone;
        const uint32_t k1 = lane + 32 < n ? keys[lo + 32 + lane] : kNone;
        const uint32_t v0 = lane < n ? vals[lo + lane] : 0u;
        const uint32_t v1 = lane + 32 < n ? vals[lo + 32 + lane] : 0u;
        const uint32_t kfirst = __shfl_sync(0xffffffffu, k0, 0);
        const bool from_before = lo > 0 && keys[lo - 1] == kfirst;
        const uint32_t key_next = lo + n < p.N ? keys[lo + n] : kNone;

        // Per entry (lane and lane + 32): does a piece end there, and what
        // becomes of it: added to d_tables (complete), carried into the next
        // chunk (cont_b), or the tail of a segment from earlier chunks (cont_a).
        uint32_t endm[2], compm[2], contbm[2];
        const uint32_t k32 = __shfl_sync(0xffffffffu, k1, 0);   // key of entry 32
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int e = lane + 32 * h;
            const uint32_t ke = h ? k1 : k0;
            const uint32_t up = __shfl_down_sync(0xffffffffu, ke, 1);
            const uint32_t nk = e + 1 < n ? (lane < 31 ? up : k32) : key_next;
            const bool valid = e < n;
            const bool end = valid && (e == n - 1 || nk != ke);
            const bool contb = end && e == n - 1 && key_next == ke;
            const bool conta = end && !contb && from_before && ke == kfirst;
            const bool comp = end && !contb && !conta && ke < p.R;
            endm[h] = __ballot_sync(0xffffffffu, end);
            compm[h] = __ballot_sync(0xffffffffu, comp);
            contbm[h] = __ballot_sync(0xffffffffu, contb);
        }

        double2 acc[PPL];
#pragma unroll
        for (int m = 0; m < PPL; ++m) acc[m] = make_double2(0.0, 0.0);
        for (int b = 0; b < n; b += BATCH) {
            __nv_bfloat162 buf[BATCH][PPL];
            float2 old[BATCH][PPL];
#pragma unroll
            for (int u = 0; u < BATCH; ++u) {
                const int e = b + u;
                const uint32_t key = lane_key(k0, k1, e);
                const uint32_t pos = __shfl_sync(0xffffffffu, e < 32 ? v0 : v1, e & 31);
                const bool use = e < n && key < p.R;
                const bool comp = e < n && ((compm[e >> 5] >> (e & 31)) & 1u);
                const __nv_bfloat162 *src = d_rows + (int64_t)pos * npairs;
                const float2 *dst = d_tables + (int64_t)key * npairs;
#pragma unroll
                for (int m = 0; m < PPL; ++m) {
                    const int j = lane + 32 * m;
                    buf[u][m] = __floats2bfloat162_rn(0.f, 0.f);
                    old[u][m] = make_float2(0.f, 0.f);
                    if (use && j < npairs) buf[u][m] = src[j];
                    if (comp && j < npairs) old[u][m] = dst[j];
                }
            }
#pragma unroll
            for (int u = 0; u < BATCH; ++u) {
                const int e = b + u;
                if (e >= n) break;
#pragma unroll
                for (int m = 0; m < PPL; ++m) {
                    const float2 f = __bfloat1622float2(buf[u][m]);
                    acc[m].x += (double)f.x;
                    acc[m].y += (double)f.y;
                }
                if (!((endm[e >> 5] >> (e & 31)) & 1u)) continue;
                const uint32_t key = lane_key(k0, k1, e);
                if ((compm[e >> 5] >> (e & 31)) & 1u) {
                    float2 *dst = d_tables + (int64_t)key * npairs;
#pragma unroll
                    for (int m = 0; m < PPL; ++m) {
                        const int j = lane + 32 * m;
                        if (j < npairs)
                            dst[j] = make_float2((float)((double)old[u][m].x + acc[m].x),
                                                 (float)((double)old[u][m].y + acc[m].y));
                    }
                } else if (key < p.R) {
                    double2 *cr = ((contbm[e >> 5] >> (e & 31)) & 1u ? carry_b : carry_a) +
                                  c * npairs;
#pragma unroll
                    for (int m = 0; m < PPL; ++m) {
                        const int j = lane + 32 * m;
                        if (j < npairs) cr[j] = acc[m];
                    }
                }
#pragma unroll
                for (int m = 0; m < PPL; ++m) acc[m] = make_double2(0.0, 0.0);
            }
        }
    }
}

// Segments that cross chunk boundaries: the warp of the chunk in which such a
// segment ends finds the chunk where it starts (a ballot over up to 32
// preceding chunk boundaries at a time), adds carry_b of every chunk from
// there up to its own, then its own carry_a, in chunk order, and updates the
// row.
template <int PPL>
__global__ void __launch_bounds__(kSegThreads)
gbwd_carry_kernel(const uint32_t *__restrict__ keys, const __grid_constant__ GatherBwdParams p,
                  float2 *__restrict__ d_tables, const double2 *__restrict__ carry_a,
                  const double2 *__restrict__ carry_b)
{
    const int lane = threadIdx.x & 31;
    const int npairs = p.D >> 1;
    const int64_t nchunks = (p.N + kSegChunk - 1) / kSegChunk;
    const int64_t nwarps = (int64_t)gridDim.x * (kSegThreads / 32);
    for (int64_t c = ((int64_t)blockIdx.x * kSegThreads + threadIdx.x) >> 5; c < nchunks;
         c += nwarps) {
        if (c == 0) continue;
        const int64_t lo = c * kSegChunk;
        const uint32_t key0 = keys[lo];
        if (keys[lo - 1] != key0 || key0 >= p.R) continue;
        const int64_t hi = min(p.N, lo + kSegChunk);
        if (hi < p.N && keys[hi] == key0) continue;   // the segment ends in a later chunk
        // first chunk of the segment: the largest j < c with keys[j * kSegChunk - 1] != key0
        // (or j = 0)
        int64_t j0 = -1;
        for (int64_t top = c - 1; j0 < 0; top -= 32) {
            const int64_t j = top - lane;
            const bool starts = j <= 0 || keys[j * kSegChunk - 1] != key0;
            const uint32_t m = __ballot_sync(0xffffffffu, starts);
            if (m) j0 = top - (__ffs(m) - 1);
        }
        double2 acc[PPL];
#pragma unroll
        for (int m = 0; m < PPL; ++m) acc[m] = make_double2(0.0, 0.0);
        for (int64_t j = j0; j <= c; ++j) {
            const double2 *src = (j < c ? carry_b : carry_a) + j * npairs;
#pragma unroll
            for (int m = 0; m < PPL; ++m) {
                const int col = lane + 32 * m;
                if (col < npairs) {
                    const double2 t = src[col];
                    acc[m].x += t.x;
                    acc[m].y += t.y;
                }
            }
        }
        float2 *dst = d_tables + (int64_t)key0 * npairs;
#pragma unroll
        for (int m = 0; m < PPL; ++m) {
            const int col = lane + 32 * m;
            if (col < npairs) {
                const float2 o = dst[col];
                dst[col] = make_float2((float)((double)o.x + acc[m].x), (float)((double)o.y + acc[m].y));
            }
        }
    }
}

}  // namespace engram
