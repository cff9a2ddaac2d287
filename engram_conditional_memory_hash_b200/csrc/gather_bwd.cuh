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
//      pass: a per-tile digit histogram, an exclusive scan of each digit's
//      counts over the tiles, and a scatter whose within-tile ranks come from
//      __match_any_sync (stable: entries keep their position order);
//   3. the sorted entries are cut into fixed chunks of kSegChunk, one warp per
//      chunk.  Each run of equal keys (a segment: all the gradients of one
//      table row, in position order) is summed in fp64 by one group of lanes
//      (each lane owns 8 columns, one 16-byte vector of the bf16 row); a
//      segment that lies inside one chunk is added to d_tables at once, a
//      segment that crosses chunk boundaries leaves one fp64 partial per chunk
//      (carry_b for the piece that continues into the next chunk, carry_a for
//      the last piece), and a second kernel adds those partials in chunk order.
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
constexpr int kSortRounds = 4;
constexpr int kSortTile = kSortThreads * kSortRounds;   // entries per CTA tile
constexpr int kRadixBins = 256;
constexpr int kScanThreads = 256;
constexpr int kSegChunk = 64;                           // sorted entries per warp
constexpr int kSegThreads = 256;
constexpr int kCarryThreads = 256;
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

// Digit histogram of one tile: hist[digit * ntiles + tile].  Every key of the
// tile is loaded before any is counted.
template <bool FROM_IDX>
__global__ void __launch_bounds__(kSortThreads)
gbwd_hist_kernel(const int64_t *__restrict__ idx, const uint32_t *__restrict__ keys,
                 const __grid_constant__ GatherBwdParams p, int shift, uint32_t *__restrict__ hist,
                 uint32_t *__restrict__ carry_count)
{
    __shared__ uint32_t sh[kRadixBins];
    const int tid = threadIdx.x;
    sh[tid] = 0;
    pdl_wait_and_release();
    if (carry_count != nullptr && blockIdx.x == 0 && tid == 0) *carry_count = 0u;
    const int64_t base = (int64_t)blockIdx.x * kSortTile;
    uint32_t kk[kSortRounds];
#pragma unroll
    for (int r = 0; r < kSortRounds; ++r) {
        const int64_t e = base + r * kSortThreads + tid;
        kk[r] = 0;
        if (e < p.N) kk[r] = FROM_IDX ? gbwd_key(idx, e, p, true) : keys[e];
    }
    __syncthreads();
#pragma unroll
    for (int r = 0; r < kSortRounds; ++r) {
        const int64_t e = base + r * kSortThreads + tid;
        if (e < p.N) atomicAdd(&sh[(kk[r] >> shift) & 0xffu], 1u);
    }
    __syncthreads();
    hist[(int64_t)tid * gridDim.x + blockIdx.x] = sh[tid];
}

// CTA d: exclusive prefix sum of digit d's tile counts hist[d * ntiles ...]
// in place, and the digit's total in totals[d].
__global__ void __launch_bounds__(kScanThreads)
gbwd_digit_scan_kernel(uint32_t *__restrict__ hist, int64_t ntiles, uint32_t *__restrict__ totals)
{
    __shared__ uint32_t warp_sum[kScanThreads / 32];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    pdl_wait_and_release();
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

// Stable scatter of one tile by the digit at `shift`.  Round r handles
// entries base + r * kSortThreads + tid, so (round, warp, lane) is position
// order.  Within a warp the rank among equal digits comes from
// __match_any_sync; across the warps of a round, from per-warp digit counts
// tagged with the round (no clearing between rounds); across rounds, from the
// running digit offsets in run[], which start at the digit's base (the sum of
// all smaller digits' totals) plus this tile's scanned count.
template <bool FROM_IDX>
__global__ void __launch_bounds__(kSortThreads)
gbwd_scatter_kernel(const int64_t *__restrict__ idx, const uint32_t *__restrict__ keys_in,
                    const uint32_t *__restrict__ vals_in, const __grid_constant__ GatherBwdParams p,
                    int shift, const uint32_t *__restrict__ hist,
                    const uint32_t *__restrict__ totals, uint32_t *__restrict__ keys_out,
                    uint32_t *__restrict__ vals_out)
{
    __shared__ uint32_t run[kRadixBins];
    __shared__ uint32_t wcnt[kSortWarps][kRadixBins];
    __shared__ uint32_t warp_sum[kSortWarps];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t base = (int64_t)blockIdx.x * kSortTile;
    pdl_wait_and_release();

    uint32_t kk[kSortRounds], vv[kSortRounds];
#pragma unroll
    for (int r = 0; r < kSortRounds; ++r) {
        const int64_t e = base + r * kSortThreads + tid;
        kk[r] = 0;
        vv[r] = 0;
        if (e < p.N) {
            if (FROM_IDX) {
                kk[r] = gbwd_key(idx, e, p, false);
                vv[r] = (uint32_t)e;
            } else {
                kk[r] = keys_in[e];
                vv[r] = vals_in[e];
            }
        }
    }

    // digit base: exclusive prefix of the digit totals (thread tid = digit)
    {
        const uint32_t t = totals[tid];
        uint32_t inc = t;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t u = __shfl_up_sync(0xffffffffu, inc, o);
            if (lane >= o) inc += u;
        }
        if (lane == 31) warp_sum[warp] = inc;
        for (int i = tid; i < kSortWarps * kRadixBins; i += kSortThreads) (&wcnt[0][0])[i] = 0u;
        __syncthreads();
        uint32_t before = 0;
        for (int w = 0; w < warp; ++w) before += warp_sum[w];
        run[tid] = before + inc - t + hist[(int64_t)tid * gridDim.x + blockIdx.x];
        __syncthreads();
    }

    const uint32_t below = (1u << lane) - 1u;
#pragma unroll
    for (int r = 0; r < kSortRounds; ++r) {
        const int64_t e = base + r * kSortThreads + tid;
        const bool valid = e < p.N;
        const uint32_t d = valid ? (kk[r] >> shift) & 0xffu : (uint32_t)kRadixBins;
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
                keys_out[pos] = kk[r];
                vals_out[pos] = vv[r];
            } else {
                record_device_error(kErrIndexRange);
            }
        }
        __syncthreads();
        if (valid && leader) atomicAdd(&run[d], (uint32_t)__popc(peers));
    }
}

// ------------------------------------------------- segmented reduction ----

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
// columns [8 cv, 8 cv + 8) of the row.  Each group loads the first gradient
// row of U segments, and the current d_tables rows of those that complete in
// this chunk, before it adds anything, so a warp keeps U * 32 / LPR random
// row reads (plus their table rows) in flight.  A row read once is finished
// from those registers; a row read several times is summed afterwards, its
// gradients loaded four at a time, so the fp64 accumulators of that rarer case
// do not add to the registers of the common one.
template <int LPR, int U>
__global__ void __launch_bounds__(kSegThreads, 3)
gbwd_segment_kernel(const uint32_t *__restrict__ keys, const uint32_t *__restrict__ vals,
                    const uint4 *__restrict__ d_rows, const __grid_constant__ GatherBwdParams p,
                    float4 *__restrict__ d_tables, double *__restrict__ carry_a,
                    double *__restrict__ carry_b, uint32_t *__restrict__ carry_list,
                    uint32_t *__restrict__ carry_count)
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
    const int64_t nchunks = (p.N + kSegChunk - 1) / kSegChunk;
    const int64_t nwarps = (int64_t)gridDim.x * kWarps;
    pdl_wait_and_release();
    for (int64_t c = ((int64_t)blockIdx.x * kSegThreads + threadIdx.x) >> 5; c < nchunks;
         c += nwarps) {
        const int64_t lo = c * kSegChunk;
        const int n = (int)min((int64_t)kSegChunk, p.N - lo);
        const uint32_t k0 = lane < n ? keys[lo + lane] : kNone;
        const uint32_t k1 = lane + 32 < n ? keys[lo + 32 + lane] : kNone;
        s_key[warp][lane] = k0;
        s_key[warp][lane + 32] = k1;
        s_pos[warp][lane] = lane < n ? vals[lo + lane] : 0u;
        s_pos[warp][lane + 32] = lane + 32 < n ? vals[lo + 32 + lane] : 0u;
        const bool from_before = lo > 0 && keys[lo - 1] == __shfl_sync(0xffffffffu, k0, 0);
        const uint32_t key_next = lo + n < p.N ? keys[lo + n] : kNone;
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
            // rows read several times: fp64 sum of all their gradients (the
            // first row and the table row are reloaded, from cache)
#pragma unroll 1
            for (int u = 0; u < U; ++u) {
                if (!multi[u]) continue;
                const int b = s_start[warp][i0 + u * GPW + grp];
                const int e_end = s_start[warp][i0 + u * GPW + grp + 1];
                double a[8] = {0.0, 0.0, 0.0, 0.0, 0.0, 0.0, 0.0, 0.0};
                for (int e = b; e < e_end; e += 4) {
                    uint4 q[4];
#pragma unroll
                    for (int x = 0; x < 4; ++x)
                        q[x] = e + x < e_end ? __ldg(d_rows + (int64_t)s_pos[warp][e + x] * nv + cv)
                                             : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
                    for (int x = 0; x < 4; ++x) add_bf16x8(a, q[x]);
                }
                const uint32_t k = s_key[warp][b];
                if (comp[u]) {
                    float4 *t = d_tables + (int64_t)k * (2 * nv) + 2 * cv;
                    const float4 x0 = t[0], x1 = t[1];
                    t[0] = make_float4((float)((double)x0.x + a[0]), (float)((double)x0.y + a[1]),
                                       (float)((double)x0.z + a[2]), (float)((double)x0.w + a[3]));
                    t[1] = make_float4((float)((double)x1.x + a[4]), (float)((double)x1.y + a[5]),
                                       (float)((double)x1.z + a[6]), (float)((double)x1.w + a[7]));
                } else {
                    double2 *cr = reinterpret_cast<double2 *>((contb[u] ? carry_b : carry_a) +
                                                              c * p.D + 8 * cv);
#pragma unroll
                    for (int x = 0; x < 4; ++x) cr[x] = make_double2(a[2 * x], a[2 * x + 1]);
                    if (!contb[u] && cv == 0) carry_list[atomicAdd(carry_count, 1u)] = (uint32_t)c;
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
// chunk c, in chunk order, and updates the row.  Each listed chunk is handled
// the same way whatever the list order, so the result stays deterministic.
__global__ void __launch_bounds__(kCarryThreads)
gbwd_carry_kernel(const uint32_t *__restrict__ keys, const __grid_constant__ GatherBwdParams p,
                  float *__restrict__ d_tables, const double *__restrict__ carry_a,
                  const double *__restrict__ carry_b, const uint32_t *__restrict__ carry_list,
                  const uint32_t *__restrict__ carry_count)
{
    pdl_wait_and_release();
    const int lane = threadIdx.x & 31;
    const int64_t count = *carry_count;
    const int64_t nwarps = (int64_t)gridDim.x * (kCarryThreads / 32);
    for (int64_t w = ((int64_t)blockIdx.x * kCarryThreads + threadIdx.x) >> 5; w < count;
         w += nwarps) {
        const int64_t cc = carry_list[w];
        const uint32_t k = keys[cc * kSegChunk];
        int64_t j0 = -1;   // the largest j < cc with keys[j * kSegChunk - 1] != k (or j = 0)
        for (int64_t top = cc - 1; j0 < 0; top -= 32) {
            const int64_t j = top - lane;
            const bool starts = j <= 0 || keys[j * kSegChunk - 1] != k;
            const uint32_t m = __ballot_sync(0xffffffffu, starts);
            if (m) j0 = top - (__ffs(m) - 1);
        }
        for (int col = lane; col < p.D; col += 32) {
            double acc = 0.0;
            for (int64_t j = j0; j < cc; j += 8) {   // 8 loads in flight, added in chunk order
                double t[8];
#pragma unroll
                for (int x = 0; x < 8; ++x) t[x] = j + x < cc ? carry_b[(j + x) * p.D + col] : 0.0;
#pragma unroll
                for (int x = 0; x < 8; ++x) acc += t[x];
            }
            acc += carry_a[cc * p.D + col];
            float *t = d_tables + (int64_t)k * p.D + col;
            *t = (float)((double)*t + acc);
        }
    }
}

}  // namespace engram
