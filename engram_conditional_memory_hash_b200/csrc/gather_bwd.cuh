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
// Entry e = t * LJ + q has the key row0(q) + idx[e], its global row (an index
// outside its table has no key: the entry is skipped and the kernels record
// ENGRAM_DEVICE_ERR_INDEX_RANGE instead of trapping).  Most rows are read by
// one entry only, and a row with one contributor needs no ordering, so:
//   1. mark: one bit per row in `seen`; an entry that finds its bit already set
//      sets the row's bit in `dupmap` (which entry arrives first does not
//      matter: a row ends up in dupmap exactly when two or more entries read it);
//   2. unique: entries whose row is not in dupmap update their row directly
//      with one rounding: fp32((double)d_tables[r] + g).  This is the
//      bandwidth-bound part; the list kernels below (stage, sort, segments,
//      carries) run beside it on a stream of higher priority (they touch only
//      rows in dupmap, it only the others);
//      stage: each tile of entries stages the (key, e) pairs of its entries
//      whose row is in dupmap, in position order, with their count and
//      first-digit histogram;
//   3. a stable least-significant-digit radix sort of the staged entries by
//      key, 8 bits per pass: a per-tile digit histogram, an exclusive scan of
//      each digit's counts over the tiles, and a scatter whose within-tile
//      ranks come from __match_any_sync (stable: entries keep their position
//      order), written out digit run by digit run.  The first pass reads the
//      staged tiles, whatever their counts; it and the later passes write the
//      list contiguously;
//   4. the sorted list is cut into fixed chunks of kSegChunk, one warp per
//      chunk.  Each run of equal keys (a segment: all the gradients of one
//      table row, in position order) is summed in fp64 by one group of lanes
//      (each lane owns 8 columns, one 16-byte vector of the bf16 row); a
//      segment that lies inside one chunk is added to d_tables at once, a
//      segment that crosses chunk boundaries leaves one fp64 partial per chunk
//      (carry_b for the piece that continues into the next chunk, carry_a for
//      the last piece), and a last kernel adds those partials in chunk order.
// Every sum has a fixed order, so the result is bitwise reproducible.  bf16
// gradients enter the fp64 sums exactly; the row's fp32 value is updated with
// one rounding: d_tables[r] = fp32((double)d_tables[r] + sum).
//
// The length M of the list exists only on the device, so the list kernels'
// grids are fixed on the host (sized for the worst case, M = N, or capped and
// looping over the work) and read M first: CTAs and warps beyond it return at
// once.
#pragma once

#include "common.cuh"
#include "hash_gather.cuh"

namespace engram {

constexpr unsigned kErrIndexRange = 2u;   // ENGRAM_DEVICE_ERR_INDEX_RANGE

constexpr int kSortThreads = 256;
constexpr int kSortWarps = kSortThreads / 32;
constexpr int kSortRounds = 4;
constexpr int kSortTile = kSortThreads * kSortRounds;   // list entries per CTA tile
constexpr int kRadixBins = 256;
constexpr int kScanThreads = 256;
constexpr int kSegChunk = 64;                           // sorted entries per warp
constexpr int kSegThreads = 256;
constexpr int kCarryThreads = 256;
constexpr int kMarkThreads = 128;
constexpr int kUniqThreads = 256;                       // staging kernel
constexpr int kUniqWarpEntries = 128;                   // entries per warp in unique/stage
constexpr int kUniqTile = kUniqThreads / 32 * kUniqWarpEntries;
constexpr int kUpdThreads = 64;                         // unique-row update
constexpr int kUpdWarpEntries = 32;                     // entries per warp in the update
constexpr int kUpdTile = kUpdThreads / 32 * kUpdWarpEntries;
static_assert(kSortThreads == kRadixBins, "one thread per digit in the histogram epilogue");
static_assert(kUniqTile == kSortTile, "the first radix pass reads the stage kernel's tiles");

struct GatherBwdParams {
    int64_t N;                          // entries: T * L * J
    int32_t LJ;                         // tables
    uint64_t lj_inv;                    // floor(2^64 / LJ) + 1 (LJ > 1): e / LJ = umulhi(e, lj_inv), e < 2^32
    int32_t D;                          // row width in bf16 values (even)
    uint32_t R;                         // rows of all tables
    uint32_t P[kHashMaxTables];         // rows of table q
    uint32_t row0[kHashMaxTables];      // first global row of table q
};

// Global row of entry e, or p.R when its index lies outside its table.
__device__ __forceinline__ uint32_t gbwd_key(const int64_t *__restrict__ idx, int64_t e,
                                             const GatherBwdParams &p, bool record)
{
    const uint32_t e32 = (uint32_t)e;   // entries < 2^30
    const int q = p.LJ == 1 ? 0 : (int)(e32 - (uint32_t)__umul64hi((uint64_t)e32, p.lj_inv) * (uint32_t)p.LJ);
    const int64_t r = __ldg(idx + e);
    if (r < 0 || r >= (int64_t)p.P[q]) {
        if (record) record_device_error(kErrIndexRange);
        return p.R;
    }
    return p.row0[q] + (uint32_t)r;
}

// Ask L2 for the `bytes` bytes at p (every 128-byte line they touch).
__device__ __forceinline__ void prefetch_l2(const void *p, uint32_t bytes)
{
    const char *c = static_cast<const char *>(p);
    for (uint32_t off = 0; off < bytes; off += 128)
        asm volatile("prefetch.global.L2 [%0];" ::"l"(c + off));
    if (bytes % 128 != 0) asm volatile("prefetch.global.L2 [%0];" ::"l"(c + bytes - 1));
}

__device__ __forceinline__ bool row_bit(const uint32_t *__restrict__ map, uint32_t key)
{
    return (map[key >> 5] >> (key & 31u)) & 1u;
}

// The same, read through L2 only (for a kernel that does not wait for its
// predecessor: the bitmap was written two kernels earlier).
__device__ __forceinline__ bool row_bit_l2(const uint32_t *__restrict__ map, uint32_t key)
{
    return (__ldcg(map + (key >> 5)) >> (key & 31u)) & 1u;
}

// ------------------------------------------------------- mark and unique ----

// seen/dupmap bits of every entry's row (both bitmaps zeroed before the
// launch): an entry that finds its row's `seen` bit already set sets the row's
// `dupmap` bit.  Which entry arrives first does not matter: a row ends up in
// dupmap exactly when two or more entries read it.  (Reading dupmap first to
// skip the atomics of hot rows saves nothing: every entry is in flight at
// once, so the check sees the bitmap before any atomic has landed.)  One
// entry per thread, in 128-thread CTAs, several waves of them: 148.0 us per
// call against 151.8 with four entries per thread (149.8 with two, 153.6 with
// eight; 256- and 512-thread CTAs 148.5 and 149.5).
__global__ void __launch_bounds__(kMarkThreads)
gbwd_mark_kernel(const int64_t *__restrict__ idx, const __grid_constant__ GatherBwdParams p,
                 uint32_t *__restrict__ seen, uint32_t *__restrict__ dupmap)
{
    pdl_wait_and_release();
    const int64_t stride = (int64_t)gridDim.x * kMarkThreads;
    for (int64_t e = (int64_t)blockIdx.x * kMarkThreads + threadIdx.x; e < p.N; e += stride) {
        const uint32_t key = gbwd_key(idx, e, p, true);
        if (key >= p.R) continue;
        const uint32_t bit = 1u << (key & 31u);
        if (atomicOr(&seen[key >> 5], bit) & bit) atomicOr(&dupmap[key >> 5], bit);
    }
}

// Rows read by one entry only: d_tables[r] = fp32((double)d_tables[r] + g).
// CTA b handles the tiles b, b + gridDim.x, ... of kUpdTile entries (one
// tile per CTA as launched, so that CTAs are short-lived and the list
// kernels, on a stream of higher priority, get SM slots as they finish:
// per call, 64-entry CTAs of 64 threads took 157 us, 128-entry ones 166,
// 256-entry ones 178, 1024-entry ones of 256 threads 181); warp w of a tile
// handles kUpdWarpEntries entries in rounds of 32 (lane l: the round's entry
// l); a round's unique entries are dealt to the warp's 32 / LPR groups of
// LPR lanes, U at a time per group, lane cv owning the columns
// [8 cv, 8 cv + 8).  32 warps per SM at 60 registers; U = 2 rows in flight
// per group (157 us per call) beat U = 1 (163-168) and U = 4 (160).
template <int LPR, int U>
__global__ void __launch_bounds__(kUpdThreads, 1024 / kUpdThreads)
gbwd_unique_kernel(const int64_t *__restrict__ idx, const uint4 *__restrict__ d_rows,
                   const __grid_constant__ GatherBwdParams p, const uint32_t *__restrict__ dupmap,
                   float4 *__restrict__ d_tables)
{
    constexpr int GPW = 32 / LPR;
    constexpr int RW = kUpdWarpEntries / 32;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int grp = lane / LPR, cv = lane % LPR;
    const int nv = p.D >> 3;
    const bool col = cv < nv;
    pdl_wait_and_release();
    const int64_t ntiles = (p.N + kUpdTile - 1) / kUpdTile;
    for (int64_t tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
        const int64_t base = tile * kUpdTile + (int64_t)warp * kUpdWarpEntries;
#pragma unroll
        for (int r = 0; r < RW; ++r) {
            const int64_t e = base + r * 32 + lane;
            const uint32_t key = e < p.N ? gbwd_key(idx, e, p, false) : p.R;
            const bool uniq = key < p.R && !row_bit(dupmap, key);
            const uint32_t um = __ballot_sync(0xffffffffu, uniq);
            if (um == 0u) continue;
            for (int j0 = 0; j0 < 32; j0 += GPW * U) {
                uint4 g[U];
                float4 o0[U], o1[U];
                uint32_t k[U];
                bool on[U];
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    const int j = j0 + u * GPW + grp;
                    k[u] = __shfl_sync(0xffffffffu, key, j);
                    on[u] = ((um >> j) & 1u) && col;
                    if (on[u]) {
                        g[u] = __ldg(d_rows + (base + r * 32 + j) * nv + cv);
                        const float4 *t = d_tables + (int64_t)k[u] * (2 * nv) + 2 * cv;
                        o0[u] = t[0];
                        o1[u] = t[1];
                    }
                }
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    if (!on[u]) continue;
                    float4 *t = d_tables + (int64_t)k[u] * (2 * nv) + 2 * cv;
                    t[0] = make_float4((float)((double)o0[u].x + (double)bf16_lo(g[u].x)),
                                       (float)((double)o0[u].y + (double)bf16_hi(g[u].x)),
                                       (float)((double)o0[u].z + (double)bf16_lo(g[u].y)),
                                       (float)((double)o0[u].w + (double)bf16_hi(g[u].y)));
                    t[1] = make_float4((float)((double)o1[u].x + (double)bf16_lo(g[u].z)),
                                       (float)((double)o1[u].y + (double)bf16_hi(g[u].z)),
                                       (float)((double)o1[u].z + (double)bf16_lo(g[u].w)),
                                       (float)((double)o1[u].w + (double)bf16_hi(g[u].w)));
                }
            }
        }
    }
}

// The entries of rows in dupmap, staged for the sort in position order: tile t
// (entries [t * kUniqTile, (t + 1) * kUniqTile)) writes their (key, e) pairs to
// stage_keys/stage_vals[t * kUniqTile ...], their count to tile_cnt[t], the
// histogram of their lowest 8 key bits to hist[digit * ntiles + t] (the first
// radix pass reads the staged tiles directly), and adds the count to *m_out,
// the length of the list.
// It runs beside the unique-row update (on another stream), after the mark
// kernel; it reads dupmap through L2.
__global__ void __launch_bounds__(kUniqThreads)
gbwd_stage_kernel(const int64_t *__restrict__ idx, const __grid_constant__ GatherBwdParams p,
                  const uint32_t *__restrict__ dupmap, uint32_t *__restrict__ stage_keys,
                  uint32_t *__restrict__ stage_vals, uint32_t *__restrict__ tile_cnt,
                  uint32_t *__restrict__ hist, uint32_t *__restrict__ m_out)
{
    constexpr int RW = kUniqWarpEntries / 32;
    __shared__ uint32_t warp_cnt[kUniqThreads / 32];
    __shared__ uint32_t sh[kRadixBins];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    sh[threadIdx.x] = 0u;
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const int64_t base = (int64_t)blockIdx.x * kUniqTile + (int64_t)warp * kUniqWarpEntries;
    uint32_t key[RW], dmask[RW];
    uint32_t ndup = 0;
#pragma unroll
    for (int r = 0; r < RW; ++r) {
        const int64_t e = base + r * 32 + lane;
        key[r] = e < p.N ? gbwd_key(idx, e, p, false) : p.R;
        dmask[r] = __ballot_sync(0xffffffffu, key[r] < p.R && row_bit_l2(dupmap, key[r]));
        ndup += (uint32_t)__popc(dmask[r]);
    }
    if (lane == 0) warp_cnt[warp] = ndup;
    __syncthreads();
    uint32_t off = 0, tot = 0;
    for (int w = 0; w < kUniqThreads / 32; ++w) {
        if (w < warp) off += warp_cnt[w];
        tot += warp_cnt[w];
    }
    if (tot != 0u) {
        const int64_t tbase = (int64_t)blockIdx.x * kUniqTile;
        const uint32_t below = (1u << lane) - 1u;
#pragma unroll
        for (int r = 0; r < RW; ++r) {
            if ((dmask[r] >> lane) & 1u) {
                const uint32_t pos = off + (uint32_t)__popc(dmask[r] & below);
                stage_keys[tbase + pos] = key[r];
                stage_vals[tbase + pos] = (uint32_t)(base + r * 32 + lane);
                atomicAdd(&sh[key[r] & 0xffu], 1u);
            }
            off += (uint32_t)__popc(dmask[r]);
        }
    }
    __syncthreads();
    hist[(int64_t)threadIdx.x * gridDim.x + blockIdx.x] = sh[threadIdx.x];
    if (threadIdx.x == 0) {
        tile_cnt[blockIdx.x] = tot;
        if (tot != 0u) atomicAdd(m_out, tot);
    }
}

// ------------------------------------------------------------ radix sort ----

__device__ __forceinline__ int64_t list_tiles(uint32_t m)
{
    return ((int64_t)m + kSortTile - 1) / kSortTile;
}

// Digit histograms of the tiles of the list: hist[digit * ntiles + tile], with
// ntiles = ceil(M / kSortTile); CTA b takes the tiles b, b + gridDim.x, ...
// Every key of a tile is loaded before any is counted.
__global__ void __launch_bounds__(kSortThreads)
gbwd_hist_kernel(const uint32_t *__restrict__ keys, const uint32_t *__restrict__ m_dev, int shift,
                 uint32_t *__restrict__ hist)
{
    __shared__ uint32_t sh[kRadixBins];
    const int tid = threadIdx.x;
    sh[tid] = 0;
    pdl_wait_and_release();
    const uint32_t M = *m_dev;
    const int64_t ntiles = list_tiles(M);
    for (int64_t tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
        const int64_t base = tile * kSortTile;
        uint32_t kk[kSortRounds];
#pragma unroll
        for (int r = 0; r < kSortRounds; ++r) {
            const int64_t e = base + r * kSortThreads + tid;
            kk[r] = e < M ? keys[e] : 0u;
        }
        __syncthreads();
#pragma unroll
        for (int r = 0; r < kSortRounds; ++r)
            if (base + r * kSortThreads + tid < M) atomicAdd(&sh[(kk[r] >> shift) & 0xffu], 1u);
        __syncthreads();
        hist[(int64_t)tid * ntiles + tile] = sh[tid];
        sh[tid] = 0;   // the next tile's counts follow the barrier above it
    }
}

// CTA d: exclusive prefix sum of digit d's tile counts hist[d * ntiles ...]
// in place, and the digit's total in totals[d].  ntiles = staged_tiles for
// the first pass (the stage kernel's tiles), else ceil(M / kSortTile).
__global__ void __launch_bounds__(kScanThreads)
gbwd_digit_scan_kernel(uint32_t *__restrict__ hist, const uint32_t *__restrict__ m_dev,
                       int64_t staged_tiles, uint32_t *__restrict__ totals)
{
    __shared__ uint32_t warp_sum[kScanThreads / 32];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    pdl_wait_and_release();
    const int64_t ntiles = staged_tiles > 0 ? staged_tiles : list_tiles(*m_dev);
    uint32_t *row = hist + (int64_t)blockIdx.x * ntiles;
    uint32_t carry = 0;
    for (int64_t b0 = 0; b0 < ntiles; b0 += kScanThreads) {
        const int64_t b = b0 + tid;
        const uint32_t v = b < ntiles ? row[b] : 0u;
        uint32_t inc = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t t = __shfl_up_sync(0xffffffffu, inc, o);
            if (lane >= o) inc += t;
        }
        if (lane == 31) warp_sum[warp] = inc;
        __syncthreads();
        uint32_t before = carry, total = 0;
#pragma unroll
        for (int w = 0; w < kScanThreads / 32; ++w) {
            const uint32_t t = warp_sum[w];
            if (w < warp) before += t;
            total += t;
        }
        if (b < ntiles) row[b] = before + inc - v;
        carry += total;
        __syncthreads();
    }
    if (tid == 0) totals[blockIdx.x] = carry;
}

// Stable scatter of the tiles of the list by the digit at `shift`; CTA b
// takes the tiles b, b + gridDim.x, ...  Round r of a tile handles entries
// base + r * kSortThreads + tid, so (round, warp, lane) is list order.  Within
// a warp the rank among equal digits comes from __match_any_sync; across the
// warps of a round, from per-warp digit counts tagged with the CTA's running
// round number (no clearing between rounds); across rounds, from running
// digit offsets.  The ranked entries are first placed in shared
// memory in digit order, then written out in that order, so that each
// digit's run of the tile goes to global memory as consecutive words: the
// run of digit d starts at the digit's base (the sum of all smaller digits'
// totals) plus this tile's scanned count.  With tile_cnt (the first pass),
// tile t of the staged_tiles tiles is the stage kernel's tile t:
// tile_cnt[t] entries from t * kSortTile on.
__global__ void __launch_bounds__(kSortThreads)
gbwd_scatter_kernel(const uint32_t *__restrict__ keys_in, const uint32_t *__restrict__ vals_in,
                    const uint32_t *__restrict__ m_dev, const uint32_t *__restrict__ tile_cnt,
                    int shift, const uint32_t *__restrict__ hist,
                    const uint32_t *__restrict__ totals, uint32_t *__restrict__ keys_out,
                    uint32_t *__restrict__ vals_out, int64_t staged_tiles)
{
    __shared__ uint32_t gbase[kRadixBins];   // global start of the tile's run of digit d
    __shared__ uint32_t lbase[kRadixBins];   // local start of that run in the tile
    __shared__ uint32_t lrun[kRadixBins];    // running local offsets while ranking
    __shared__ uint32_t wcnt[kSortWarps][kRadixBins];
    __shared__ uint32_t warp_sum[2][kSortWarps];
    __shared__ uint32_t s_key[kSortTile], s_val[kSortTile];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    lrun[tid] = 0u;
    for (int i = tid; i < kSortWarps * kRadixBins; i += kSortThreads) (&wcnt[0][0])[i] = 0u;
    pdl_wait_and_release();
    const uint32_t M = *m_dev;
    const int64_t ntiles = tile_cnt != nullptr ? staged_tiles : list_tiles(M);
    uint32_t iter = 0;
    for (int64_t tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++iter) {
        __syncthreads();   // nothing of the previous tile is read after this
        lrun[tid] = 0u;
        const int64_t base = tile * kSortTile;
        const int n = tile_cnt != nullptr ? (int)min((uint32_t)kSortTile, tile_cnt[tile])
                                          : (int)min((int64_t)kSortTile, (int64_t)M - base);
        if (n <= 0) continue;

        uint32_t kk[kSortRounds], vv[kSortRounds];
#pragma unroll
        for (int r = 0; r < kSortRounds; ++r) {
            const int e = r * kSortThreads + tid;
            kk[r] = e < n ? keys_in[base + e] : 0u;
            vv[r] = e < n ? vals_in[base + e] : 0u;
        }
        const uint32_t tot = totals[tid];
        const uint32_t tile_off = hist[(int64_t)tid * ntiles + tile];
        __syncthreads();
#pragma unroll
        for (int r = 0; r < kSortRounds; ++r)
            if (r * kSortThreads + tid < n) atomicAdd(&lrun[(kk[r] >> shift) & 0xffu], 1u);
        __syncthreads();

        // exclusive scans over the digits (thread tid = digit): of the digit
        // totals for the global base, and of this tile's counts for the local base
        {
            const uint32_t cnt = lrun[tid];
            uint32_t ig = tot, il = cnt;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const uint32_t ug = __shfl_up_sync(0xffffffffu, ig, o);
                const uint32_t ul = __shfl_up_sync(0xffffffffu, il, o);
                if (lane >= o) {
                    ig += ug;
                    il += ul;
                }
            }
            if (lane == 31) {
                warp_sum[0][warp] = ig;
                warp_sum[1][warp] = il;
            }
            __syncthreads();
            uint32_t bg = 0, bl = 0;
            for (int w = 0; w < warp; ++w) {
                bg += warp_sum[0][w];
                bl += warp_sum[1][w];
            }
            gbase[tid] = bg + ig - tot + tile_off;
            lbase[tid] = bl + il - cnt;
            lrun[tid] = bl + il - cnt;
            __syncthreads();
        }

        const uint32_t below = (1u << lane) - 1u;
#pragma unroll
        for (int r = 0; r < kSortRounds; ++r) {
            const bool valid = r * kSortThreads + tid < n;
            const uint32_t d = valid ? (kk[r] >> shift) & 0xffu : (uint32_t)kRadixBins;
            const uint32_t peers = __match_any_sync(0xffffffffu, d);
            const bool leader = (__ffs(peers) - 1) == lane;
            const uint32_t tag = (iter * (uint32_t)kSortRounds + (uint32_t)r + 1u) << 8;
            if (valid && leader) wcnt[warp][d] = tag | (uint32_t)__popc(peers);
            __syncthreads();
            if (valid) {
                uint32_t lp = lrun[d] + (uint32_t)__popc(peers & below);
                for (int w = 0; w < warp; ++w) {
                    const uint32_t c = wcnt[w][d];
                    if ((c & ~0xffu) == tag) lp += c & 0xffu;
                }
                s_key[lp] = kk[r];   // lp < n: the local counts are this tile's own
                s_val[lp] = vv[r];
            }
            __syncthreads();
            if (valid && leader) atomicAdd(&lrun[d], (uint32_t)__popc(peers));
        }
        __syncthreads();
        for (int i = tid; i < n; i += kSortThreads) {
            const uint32_t k = s_key[i];
            const uint32_t d = (k >> shift) & 0xffu;
            const uint32_t pos = gbase[d] + ((uint32_t)i - lbase[d]);
            // pos < M whenever the histogram counted the same keys; the check only
            // keeps every write inside the buffers if that ever failed
            if (pos < M) {
                keys_out[pos] = k;
                vals_out[pos] = s_val[i];
            } else {
                record_device_error(kErrIndexRange);
            }
        }
    }
}

// ------------------------------------------------- segmented reduction ----

constexpr int kLongRun = 16;   // runs longer than this are summed by the whole warp

// The end of a segment piece summed into a[8] (this lane's 8 columns):
// completes the row (comp) with one rounding, or leaves the partial for the
// carry kernel (carry_b if the segment continues into the next chunk, else
// carry_a, listing the chunk).
__device__ __forceinline__ void finish_segment(const double a[8], bool comp, bool contb, uint32_t key,
                                               int64_t c, int cv, int nv, int D,
                                               float4 *__restrict__ d_tables,
                                               double *__restrict__ carry_a,
                                               double *__restrict__ carry_b,
                                               uint32_t *__restrict__ carry_list,
                                               uint32_t *__restrict__ carry_count)
{
    if (comp) {
        float4 *t = d_tables + (int64_t)key * (2 * nv) + 2 * cv;
        const float4 x0 = t[0], x1 = t[1];
        t[0] = make_float4((float)((double)x0.x + a[0]), (float)((double)x0.y + a[1]),
                           (float)((double)x0.z + a[2]), (float)((double)x0.w + a[3]));
        t[1] = make_float4((float)((double)x1.x + a[4]), (float)((double)x1.y + a[5]),
                           (float)((double)x1.z + a[6]), (float)((double)x1.w + a[7]));
    } else {
        double2 *cr = reinterpret_cast<double2 *>((contb ? carry_b : carry_a) + c * D + 8 * cv);
#pragma unroll
        for (int x = 0; x < 4; ++x) cr[x] = make_double2(a[2 * x], a[2 * x + 1]);
        if (!contb && cv == 0) carry_list[atomicAdd(carry_count, 1u)] = (uint32_t)c;
    }
}

// 8 bf16 values of a 16-byte vector added to 8 fp64 accumulators (exactly:
// every bf16 value is a double, and the sum rounds once per add).
__device__ __forceinline__ void add_bf16x8(double a[8], const uint4 &q)
{
    const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        a[2 * i] += (double)bf16_lo(w[i]);
        a[2 * i + 1] += (double)bf16_hi(w[i]);
    }
}

// One warp per chunk of kSegChunk sorted entries.  The chunk's keys and
// positions go to shared memory, the segment starts are found with ballots,
// and the segments are dealt to the warp's 32 / LPR groups of LPR lanes in
// order (segment i to group i mod groups); lane cv of a group owns the 8
// columns [8 cv, 8 cv + 8) of the row.  As soon as the chunk's keys are known
// the warp asks L2 for every gradient row of the chunk and every table row
// that completes in it (prefetches hold no registers), so all of the chunk's
// random row reads are in flight at once.  Each group then loads the first
// gradient row of U segments, and the current d_tables rows of those that
// complete in this chunk, before it adds anything.  A row read once is finished
// from those registers; a row read several times is summed afterwards (a long
// run of one hot row by the whole warp, the groups splitting its gradients),
// so the fp64 accumulators of that case do not add to the registers of the
// common one.  Four CTAs per SM (64 registers a thread) run faster than
// three (209 -> 206 us per call at the full-path workload), and one segment
// at a time per group (U = 1) faster than two (194 -> 191 us).
template <int LPR, int U>
__global__ void __launch_bounds__(kSegThreads, 4)
gbwd_segment_kernel(const uint32_t *__restrict__ keys, const uint32_t *__restrict__ vals,
                    const uint4 *__restrict__ d_rows, const __grid_constant__ GatherBwdParams p,
                    float4 *__restrict__ d_tables, double *__restrict__ carry_a,
                    double *__restrict__ carry_b, uint32_t *__restrict__ carry_list,
                    uint32_t *__restrict__ carry_count, const uint32_t *__restrict__ m_dev)
{
    constexpr int GPW = 32 / LPR;
    constexpr int kWarps = kSegThreads / 32;
    constexpr uint32_t kNone = 0xffffffffu;   // never a key: keys are <= R < 2^32 - 1
    __shared__ uint32_t s_key[kWarps][kSegChunk];
    __shared__ uint32_t s_pos[kWarps][kSegChunk];
    __shared__ uint8_t s_start[kWarps][kSegChunk + 4];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int grp = lane / LPR, cv = lane % LPR;
    const int nv = p.D >> 3;                  // 16-byte vectors per row
    const bool col = cv < nv;
    const int64_t nwarps = (int64_t)gridDim.x * kWarps;
    pdl_wait_and_release();
    const int64_t M = *m_dev;
    const int64_t nchunks = (M + kSegChunk - 1) / kSegChunk;
    for (int64_t c = ((int64_t)blockIdx.x * kSegThreads + threadIdx.x) >> 5; c < nchunks;
         c += nwarps) {
        const int64_t lo = c * kSegChunk;
        const int n = (int)min((int64_t)kSegChunk, M - lo);
        const uint32_t k0 = lane < n ? keys[lo + lane] : kNone;
        const uint32_t k1 = lane + 32 < n ? keys[lo + 32 + lane] : kNone;
        s_key[warp][lane] = k0;
        s_key[warp][lane + 32] = k1;
        s_pos[warp][lane] = lane < n ? vals[lo + lane] : 0u;
        s_pos[warp][lane + 32] = lane + 32 < n ? vals[lo + 32 + lane] : 0u;
        const bool from_before = lo > 0 && keys[lo - 1] == __shfl_sync(0xffffffffu, k0, 0);
        const uint32_t key_next = lo + n < M ? keys[lo + n] : kNone;
        const uint32_t k31 = __shfl_sync(0xffffffffu, k0, 31);
        const uint32_t up0 = __shfl_up_sync(0xffffffffu, k0, 1);
        const uint32_t up1 = __shfl_up_sync(0xffffffffu, k1, 1);
        const bool st0 = lane < n && (lane == 0 || k0 != up0);
        const bool st1 = lane + 32 < n && k1 != (lane == 0 ? k31 : up1);
        const uint32_t m0 = __ballot_sync(0xffffffffu, st0);
        const uint32_t m1 = __ballot_sync(0xffffffffu, st1);
        const int nseg = __popc(m0) + __popc(m1);
        const uint32_t below = (1u << lane) - 1u;
        if (st0) s_start[warp][__popc(m0 & below)] = (uint8_t)lane;
        if (st1) s_start[warp][__popc(m0) + __popc(m1 & below)] = (uint8_t)(lane + 32);
        if (lane == 0) s_start[warp][nseg] = (uint8_t)n;
        const uint32_t klast = __shfl_sync(0xffffffffu, n > 32 ? k1 : k0, (n - 1) & 31);
        const bool last_cont = key_next == klast;
        // Request every row the chunk will read before anything waits on one:
        // the gradient row of each entry, and the table row of each segment
        // that ends (and completes) here.  The loads below then hit L2.
        {
            const uint32_t kfirst = __shfl_sync(0xffffffffu, k0, 0);
            const uint32_t dn0 = __shfl_down_sync(0xffffffffu, k0, 1);
            const uint32_t dn1 = __shfl_down_sync(0xffffffffu, k1, 1);
            const uint32_t k32 = __shfl_sync(0xffffffffu, k1, 0);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int e = lane + 32 * h;
                const uint32_t ke = h ? k1 : k0;
                if (e < n && ke < p.R) {
                    // this lane wrote s_pos[warp][e] itself
                    prefetch_l2(d_rows + (int64_t)s_pos[warp][e] * nv, (uint32_t)p.D * 2u);
                    const uint32_t nk = e + 1 < n ? (h ? dn1 : (lane < 31 ? dn0 : k32)) : key_next;
                    const bool end = e == n - 1 || nk != ke;
                    const bool contb = e == n - 1 && last_cont;
                    const bool conta = from_before && ke == kfirst;
                    if (end && !contb && !conta)
                        prefetch_l2(d_tables + (int64_t)ke * (2 * nv), (uint32_t)p.D * 4u);
                }
            }
        }
        __syncwarp();

        for (int i0 = 0; i0 < nseg; i0 += GPW * U) {
            uint4 row[U];
            float4 o0[U], o1[U];
            int sb[U], se[U];
            uint32_t key[U];
            bool use[U], comp[U], contb[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int i = i0 + u * GPW + grp;
                const bool valid = i < nseg;
                sb[u] = valid ? s_start[warp][i] : 0;
                se[u] = valid ? s_start[warp][i + 1] : 0;
                key[u] = valid ? s_key[warp][sb[u]] : kNone;
                contb[u] = valid && i == nseg - 1 && last_cont;
                const bool conta = valid && i == 0 && from_before && !contb[u];
                use[u] = valid && key[u] < p.R;
                comp[u] = use[u] && !contb[u] && !conta;
                row[u] = make_uint4(0u, 0u, 0u, 0u);
                o0[u] = o1[u] = make_float4(0.f, 0.f, 0.f, 0.f);
                if (use[u] && col) row[u] = __ldg(d_rows + (int64_t)s_pos[warp][sb[u]] * nv + cv);
                if (comp[u] && col) {
                    const float4 *t = d_tables + (int64_t)key[u] * (2 * nv) + 2 * cv;
                    o0[u] = t[0];
                    o1[u] = t[1];
                }
            }
            // rows read once (almost all of them at realistic sizes): one
            // rounding of old + gradient, or the gradient as a carry
            bool multi[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                multi[u] = use[u] && col && se[u] - sb[u] > 1;
                if (!use[u] || !col || multi[u]) continue;
                const float2 g0 = make_float2(bf16_lo(row[u].x), bf16_hi(row[u].x));
                const float2 g1 = make_float2(bf16_lo(row[u].y), bf16_hi(row[u].y));
                const float2 g2 = make_float2(bf16_lo(row[u].z), bf16_hi(row[u].z));
                const float2 g3 = make_float2(bf16_lo(row[u].w), bf16_hi(row[u].w));
                if (comp[u]) {
                    float4 *t = d_tables + (int64_t)key[u] * (2 * nv) + 2 * cv;
                    t[0] = make_float4((float)((double)o0[u].x + (double)g0.x),
                                       (float)((double)o0[u].y + (double)g0.y),
                                       (float)((double)o0[u].z + (double)g1.x),
                                       (float)((double)o0[u].w + (double)g1.y));
                    t[1] = make_float4((float)((double)o1[u].x + (double)g2.x),
                                       (float)((double)o1[u].y + (double)g2.y),
                                       (float)((double)o1[u].z + (double)g3.x),
                                       (float)((double)o1[u].w + (double)g3.y));
                } else {
                    double2 *cr = reinterpret_cast<double2 *>((contb[u] ? carry_b : carry_a) +
                                                              c * p.D + 8 * cv);
                    cr[0] = make_double2(g0.x, g0.y);
                    cr[1] = make_double2(g1.x, g1.y);
                    cr[2] = make_double2(g2.x, g2.y);
                    cr[3] = make_double2(g3.x, g3.y);
                    // the last piece of a segment from earlier chunks: this
                    // chunk goes on the list the carry kernel works through
                    if (!contb[u] && cv == 0) carry_list[atomicAdd(carry_count, 1u)] = (uint32_t)c;
                }
            }
            // rows read several times.  A short run (up to kLongRun entries)
            // is summed by its own group: the first four gradients of each of
            // the group's U runs are requested together, the rest four at a
            // time;
            // a long run (a hot row) by the whole warp: group g takes the
            // entries b + g, b + g + GPW, ... (four at a time) and the groups'
            // partials are combined by a butterfly over the groups (a fixed
            // order; every group ends with the same bits).  All sums are fp64;
            // the first gradient row and the table row are reloaded, from cache.
            {
                double a[U][8];
                uint4 q[U][4];
                bool sh[U];
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    sh[u] = multi[u] && se[u] - sb[u] <= kLongRun;
#pragma unroll
                    for (int k = 0; k < 8; ++k) a[u][k] = 0.0;
#pragma unroll
                    for (int x = 0; x < 4; ++x)
                        q[u][x] = sh[u] && sb[u] + x < se[u]
                                      ? __ldg(d_rows + (int64_t)s_pos[warp][sb[u] + x] * nv + cv)
                                      : make_uint4(0u, 0u, 0u, 0u);
                }
#pragma unroll
                for (int u = 0; u < U; ++u) {
#pragma unroll
                    for (int x = 0; x < 4; ++x) add_bf16x8(a[u], q[u][x]);
                }
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    if (!sh[u]) continue;
                    for (int e = sb[u] + 4; e < se[u]; e += 4) {
                        uint4 r4[4];
#pragma unroll
                        for (int x = 0; x < 4; ++x)
                            r4[x] = e + x < se[u] ? __ldg(d_rows + (int64_t)s_pos[warp][e + x] * nv + cv)
                                                  : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
                        for (int x = 0; x < 4; ++x) add_bf16x8(a[u], r4[x]);
                    }
                    finish_segment(a[u], comp[u], contb[u], key[u], c, cv, nv, p.D, d_tables, carry_a, carry_b,
                                   carry_list, carry_count);
                }
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                uint32_t mm = __ballot_sync(0xffffffffu, multi[u] && cv == 0 && se[u] - sb[u] > kLongRun);
                while (mm) {
                    const int src = __ffs(mm) - 1;   // lane 0 of the owning group
                    mm &= mm - 1u;
                    const int b = __shfl_sync(0xffffffffu, sb[u], src);
                    const int e_end = __shfl_sync(0xffffffffu, se[u], src);
                    const bool ocomp = __shfl_sync(0xffffffffu, (int)comp[u], src) != 0;
                    const bool ocontb = __shfl_sync(0xffffffffu, (int)contb[u], src) != 0;
                    double a[8] = {0.0, 0.0, 0.0, 0.0, 0.0, 0.0, 0.0, 0.0};
                    for (int e = b + grp; e < e_end; e += 4 * GPW) {
                        uint4 q[4];
#pragma unroll
                        for (int x = 0; x < 4; ++x) {
                            const int ee = e + x * GPW;
                            q[x] = (ee < e_end && col) ? __ldg(d_rows + (int64_t)s_pos[warp][ee] * nv + cv)
                                                       : make_uint4(0u, 0u, 0u, 0u);
                        }
#pragma unroll
                        for (int x = 0; x < 4; ++x) add_bf16x8(a, q[x]);
                    }
#pragma unroll
                    for (int o = LPR; o < 32; o <<= 1) {
#pragma unroll
                        for (int k = 0; k < 8; ++k) a[k] += __shfl_xor_sync(0xffffffffu, a[k], o);
                    }
                    if (grp == 0 && col)
                        finish_segment(a, ocomp, ocontb, s_key[warp][b], c, cv, nv, p.D, d_tables, carry_a,
                                       carry_b, carry_list, carry_count);
                }
            }
        }
        __syncwarp();
    }
}

// Segments that cross chunk boundaries.  The segment kernel lists every chunk
// that holds the end of such a segment (carry_list, carry_count entries, in
// no particular order); one warp per listed chunk c finds the chunk where the
// segment starts (a ballot over up to 32 preceding chunk boundaries at a
// time), adds carry_b of every chunk from there up to chunk c, then carry_a of
// chunk c, in chunk order, and updates the row.  Lane l owns the columns
// l, l + 32, ... (MC of them); the partials of 16 / MC chunks are loaded
// before any is added.  Each listed chunk is handled the same way whatever the
// list order, so the result stays deterministic.
template <int MC>
__global__ void __launch_bounds__(kCarryThreads)
gbwd_carry_kernel(const uint32_t *__restrict__ keys, const __grid_constant__ GatherBwdParams p,
                  float *__restrict__ d_tables, const double *__restrict__ carry_a,
                  const double *__restrict__ carry_b, const uint32_t *__restrict__ carry_list,
                  const uint32_t *__restrict__ carry_count)
{
    constexpr int CB = 16 / MC;
    pdl_wait_and_release();
    const int lane = threadIdx.x & 31;
    const int64_t count = *carry_count;
    const int64_t nwarps = (int64_t)gridDim.x * (kCarryThreads / 32);
    for (int64_t w = ((int64_t)blockIdx.x * kCarryThreads + threadIdx.x) >> 5; w < count;
         w += nwarps) {
        const int64_t cc = carry_list[w];
        const uint32_t k = keys[cc * kSegChunk];
        float old[MC];
        double acc[MC];
#pragma unroll
        for (int m = 0; m < MC; ++m) {
            const int col = lane + 32 * m;
            old[m] = col < p.D ? d_tables[(int64_t)k * p.D + col] : 0.f;
            acc[m] = 0.0;
        }
        int64_t j0 = -1;   // the largest j < cc with keys[j * kSegChunk - 1] != k (or j = 0)
        for (int64_t top = cc - 1; j0 < 0; top -= 32) {
            const int64_t j = top - lane;
            const bool starts = j <= 0 || keys[j * kSegChunk - 1] != k;
            const uint32_t m = __ballot_sync(0xffffffffu, starts);
            if (m) j0 = top - (__ffs(m) - 1);
        }
        for (int64_t j = j0; j < cc; j += CB) {
            double t[CB][MC];
#pragma unroll
            for (int x = 0; x < CB; ++x) {
#pragma unroll
                for (int m = 0; m < MC; ++m) {
                    const int col = lane + 32 * m;
                    t[x][m] = (j + x < cc && col < p.D) ? carry_b[(j + x) * p.D + col] : 0.0;
                }
            }
#pragma unroll
            for (int x = 0; x < CB; ++x) {
#pragma unroll
                for (int m = 0; m < MC; ++m) acc[m] += t[x][m];
            }
        }
#pragma unroll
        for (int m = 0; m < MC; ++m) {
            const int col = lane + 32 * m;
            if (col < p.D) {
                acc[m] += carry_a[cc * p.D + col];
                d_tables[(int64_t)k * p.D + col] = (float)((double)old[m] + acc[m]);
            }
        }
    }
}

}  // namespace engram
