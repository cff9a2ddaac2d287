// Fused Engram gate, forward and backward (sm_100a).
//
// The gate of the page "DeepSeek 开源 TileKernels" (zhichai.net/topic/177618722),
// section "5. Engram — 条件记忆门控":
//     gate = sigmoid(signed_sqrt(dot(RMSNorm(x, wh), RMSNorm(k, we)) * scalar))
//     out  = x + gate * v
// written in the fused form this kernel evaluates, with w = wh * we (the
// page's "engram_fused_weight"; the product of two bf16 values is exact in
// fp32):
//     dot = rx * rk * sum_j x_j k_j w_j,  rx = (sum_j x_j^2 / H + eps)^(-1/2)
//
// Both kernels are persistent: CTA c of G handles tokens c, c+G, c+2G, ...
// A single thread streams each token's rows (x, k, v for the forward; g, x, k,
// v for the backward) from HBM into a ring of shared-memory stages with 1-D
// bulk copies (cp.async.bulk, completing on one mbarrier per stage), several
// tokens ahead of the compute.  Each thread owns the same MAXV 16-byte column
// vectors j = tid + m * blockDim.x of every token, so the fused weight and the
// backward's weight-gradient accumulators stay in registers for the whole
// kernel.  Per token: one pass over the staged rows into registers accumulates
// the statistics (sum x^2, sum k^2 and, in the backward, sum g v in fp32; the
// dot product sum x k w in fp64, see below), a warp-shuffle + shared-memory
// block reduction combines them in a fixed order, the stage is handed back to
// the copy engine (its contents now live in registers), and the outputs are
// computed from registers and written with streaming 16-byte stores.
//
// Precision.  x_j k_j is exact in fp32 and w_j is exact in fp32, so every
// term of the dot product enters the fp64 accumulator exactly (one fp64
// rounding per add).  This matters near s = 0: the backward multiplies by
// 1/(2 sqrt|s|), so fp32 rounding of a cancelling dot product would be
// magnified for tokens with tiny |s|.  The per-token scalar chain uses the
// hardware reciprocal square root, exponential and reciprocal (a few ulp,
// far inside the gate's tolerance).
#pragma once

#include "common.cuh"

namespace engram {

// Largest CTA of a gate kernel whose threads own `maxv` column vectors each
// (rows of up to 8192 values; one vector per thread caps the CTA at 512 so
// that those threads may hold 128 registers).
__host__ __device__ constexpr int gate_max_threads(int maxv) { return maxv == 1 ? 512 : 1024 / maxv; }
// Block reduction: per warp and token parity, the fp32 sums (float4) and the
// fp64 dot product (double).
constexpr size_t kGateRedBytes = 2 * 32 * sizeof(float4) + 2 * 32 * sizeof(double);

// Shared-memory bytes of a gate kernel with `nstage` stages of `ntensors` rows.
__host__ __device__ inline size_t gate_smem_bytes(int H, int ntensors, int nstage)
{
    return (size_t)nstage * (size_t)ntensors * (size_t)H * 2u  // data stages
           + kGateRedBytes                                    // block-reduction buffers
           + (size_t)nstage * 8u;                             // one mbarrier per stage
}

// Extra bytes added to every stage's expected transaction count.  Always 0 in
// the library; the pipeline-timeout test builds a copy of the library with a
// non-zero value, so that no stage ever completes and every wait runs into
// its time limit (nothing faults: the copies themselves are unchanged).
#ifndef ENGRAM_TEST_EXTRA_TX
#define ENGRAM_TEST_EXTRA_TX 0u
#endif

// Issue the bulk copies of token `row` (NTENSORS rows of row_bytes) into stage
// `s`.  Called by one thread.
template <int NTENSORS>
__device__ __forceinline__ void gate_issue_row(unsigned char *smem, uint32_t bar0,
                                               const void *const *src, int64_t row,
                                               uint32_t row_bytes, int s)
{
    const uint32_t stage_bytes = NTENSORS * row_bytes;
    const uint32_t dst = smem_addr(smem + (size_t)s * stage_bytes);
    const uint32_t bar = bar0 + 8u * (uint32_t)s;
    mbar_arrive_expect_tx(bar, stage_bytes + ENGRAM_TEST_EXTRA_TX);
#pragma unroll
    for (int q = 0; q < NTENSORS; ++q) {
        const char *p = static_cast<const char *>(src[q]) + row * (int64_t)row_bytes;
        bulk_load(dst + (uint32_t)q * row_bytes, p, row_bytes, bar);
    }
}

__device__ __forceinline__ double warp_sum_f64(double v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// After a failed wait: wait (sharing one time limit) for every copy still in
// flight into this CTA's shared memory, so that none lands after the CTA exits.
__device__ __forceinline__ void gate_drain(uint32_t bar0, int64_t i, int64_t nrows, int nstage)
{
    const uint64_t t0 = globaltimer_ns();
    const int64_t last = (i + nstage < nrows) ? i + nstage : nrows;
    for (int64_t j = i; j < last; ++j) {
        const uint32_t bar = bar0 + 8u * (uint32_t)(j % nstage);
        const uint32_t parity = (uint32_t)((j / nstage) & 1);
        while (!mbar_try_wait(bar, parity)) {
            if (globaltimer_ns() - t0 > kWaitLimitNs) return;
        }
    }
}

// Shared prologue: barriers, then the first min(nstage, nrows) tokens in flight.
template <int NTENSORS>
__device__ __forceinline__ void gate_pipeline_start(unsigned char *smem, uint32_t bar0,
                                                    const void *const *src, int64_t first,
                                                    int64_t G, int64_t nrows, uint32_t row_bytes,
                                                    int nstage)
{
    if (threadIdx.x == 0) {
        for (int s = 0; s < nstage; ++s) mbar_init(bar0 + 8u * s, 1);
        fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        const int64_t pre = nrows < nstage ? nrows : nstage;
        for (int64_t i = 0; i < pre; ++i)
            gate_issue_row<NTENSORS>(smem, bar0, src, first + i * G, row_bytes, (int)(i % nstage));
    }
}

// Sum of the per-warp partials of one token, in warp order (a fixed order):
// every thread adds the nwarps entries itself, which keeps the per-token
// critical path short (a shuffle tree over the warps' entries was measured
// slower: it lengthens the chain every token waits on).
__device__ __forceinline__ void combine_partials(const float4 *rb, const double *rbd, int nwarps,
                                                 float4 &r, double &A)
{
    r = make_float4(0.f, 0.f, 0.f, 0.f);
    A = 0.0;
    for (int q = 0; q < nwarps; ++q) {
        const float4 t = rb[q];
        r.x += t.x;
        r.y += t.y;
        r.z += t.z;
        A += rbd[q];
    }
}

// Per-token gate from the reduced statistics.
struct GateScalars {
    float rx, rk, d, s, gate;
};

__device__ __forceinline__ GateScalars gate_scalars(float Sx, float Sk, double A, float inv_h,
                                                    float eps, float scalar)
{
    GateScalars r;
    r.rx = rsqrtf(fmaf(Sx, inv_h, eps));
    r.rk = rsqrtf(fmaf(Sk, inv_h, eps));
    r.d = (r.rx * r.rk) * (float)A;
    r.s = r.d * scalar;
    const float as = fabsf(r.s);
    const float u = as > 0.f ? copysignf(as * rsqrtf(as), r.s) : 0.f;  // signed_sqrt(s)
    r.gate = __fdividef(1.0f, 1.0f + __expf(-u));
    return r;
}

// --------------------------------------------------------------- forward ----

template <int MAXV>
__global__ void __launch_bounds__(gate_max_threads(MAXV), MAXV == 4 ? 2 : 1)
gate_fwd_kernel(const uint4 *__restrict__ x, const uint4 *__restrict__ k,
                const uint4 *__restrict__ v, const uint4 *__restrict__ wh,
                const uint4 *__restrict__ we, int64_t T, int H, float eps, float scalar,
                uint4 *__restrict__ out, float *__restrict__ gate, int nstage)
{
    extern __shared__ __align__(128) unsigned char smem[];
    const int nvec = H >> 3;
    const uint32_t row_bytes = (uint32_t)H * 2u;
    const uint32_t stage_bytes = 3u * row_bytes;
    unsigned char *tail = smem + (size_t)nstage * stage_bytes;
    float4 *red = reinterpret_cast<float4 *>(tail);                              // [2][32]
    double *redd = reinterpret_cast<double *>(tail + 2 * 32 * sizeof(float4));   // [2][32]
    const uint32_t bar0 = smem_addr(tail + kGateRedBytes);

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int nthreads = blockDim.x, nwarps = nthreads >> 5;

    // fused weight of this thread's columns, kept in fp64 for the dot product
    double w[MAXV][8];
#pragma unroll
    for (int m = 0; m < MAXV; ++m) {
        const int vi = tid + m * nthreads;
        float2 a[4], b[4];
        if (vi < nvec) {
            unpack4x2(wh[vi], a);
            unpack4x2(we[vi], b);
        } else {
#pragma unroll
            for (int e = 0; e < 4; ++e) a[e] = b[e] = make_float2(0.f, 0.f);
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float2 p = __fmul2_rn(a[e], b[e]);
            w[m][2 * e] = (double)p.x;
            w[m][2 * e + 1] = (double)p.y;
        }
    }

    const int64_t G = gridDim.x, first = blockIdx.x;
    const int64_t nrows = T > first ? (T - first + G - 1) / G : 0;
    const void *src[3] = {x, k, v};
    gate_pipeline_start<3>(smem, bar0, src, first, G, nrows, row_bytes, nstage);

    const float inv_h = 1.0f / (float)H;
    for (int64_t i = 0; i < nrows; ++i) {
        const int s = (int)(i % nstage);
        const bool ok = mbar_wait_bounded(bar0 + 8u * s, (uint32_t)((i / nstage) & 1));
        const uint4 *sx = reinterpret_cast<const uint4 *>(smem + (size_t)s * stage_bytes);
        const uint4 *sk = sx + nvec;
        const uint4 *sv = sk + nvec;

        uint4 xq[MAXV], vq[MAXV];
        float2 px2 = make_float2(0.f, 0.f), pk2 = px2;
        double pa = 0.0;
#pragma unroll
        for (int m = 0; m < MAXV; ++m) {
            const int vi = tid + m * nthreads;
            if (vi < nvec) {
                xq[m] = sx[vi];
                vq[m] = sv[vi];
                float2 xf[4], kf[4];
                unpack4x2(xq[m], xf);
                unpack4x2(sk[vi], kf);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    px2 = __ffma2_rn(xf[e], xf[e], px2);
                    pk2 = __ffma2_rn(kf[e], kf[e], pk2);
                    const float2 xk = __fmul2_rn(xf[e], kf[e]);   // exact
                    pa = fma((double)xk.x, w[m][2 * e], pa);
                    pa = fma((double)xk.y, w[m][2 * e + 1], pa);
                }
            }
        }
        float px = warp_sum(px2.x + px2.y);
        float pk = warp_sum(pk2.x + pk2.y);
        pa = warp_sum_f64(pa);
        float4 *rb = red + (i & 1) * 32;
        double *rbd = redd + (i & 1) * 32;
        if (lane == 0) {
            rb[warp] = make_float4(px, pk, 0.f, 0.f);
            rbd[warp] = pa;
        }
        if (__syncthreads_or(!ok)) {
            if (tid == 0) {
                record_device_error(kErrPipelineTimeout);
                gate_drain(bar0, i, nrows, nstage);
            }
            return;
        }
        // Every thread holds its part of this token in registers: hand the
        // stage back to the copy engine.
        if (tid == 0 && i + nstage < nrows)
            gate_issue_row<3>(smem, bar0, src, first + (i + nstage) * G, row_bytes, s);

        float4 r;
        double A;
        combine_partials(rb, rbd, nwarps, r, A);
        const GateScalars c = gate_scalars(r.x, r.y, A, inv_h, eps, scalar);

        const int64_t row = first + i * G;
        uint4 *orow = out + row * nvec;
        const float2 gate2 = make_float2(c.gate, c.gate);
#pragma unroll
        for (int m = 0; m < MAXV; ++m) {
            const int vi = tid + m * nthreads;
            if (vi < nvec) {
                float2 xf[4], vf[4], of[4];
                unpack4x2(xq[m], xf);
                unpack4x2(vq[m], vf);
#pragma unroll
                for (int e = 0; e < 4; ++e) of[e] = __ffma2_rn(gate2, vf[e], xf[e]);
                __stcs(orow + vi, pack4x2(of));
            }
        }
        if (tid == 0 && gate != nullptr) gate[row] = c.gate;
    }
}

// ------------------------------------------------ weight-gradient level 2 ----
//
// P_j = sum_p w_partial[p][j] over the G partial rows, in one order fixed by G
// alone, so that the standalone reduction kernel and the tail fused into the
// backward kernel give the same bits.  The rows form `count` consecutive
// groups of `size` rows (the last one may be shorter):
//     r_q = (((0 + Q_{q*size}) + Q_{q*size+1}) + ...)      in row order
//     P   = (((0 + r_0) + r_1) + ...)                       in group order
//     dwh_j = we_j * P_j,   dwe_j = wh_j * P_j
// size = max(ceil(sqrt(G)), ceil(G / 32)), so that there are at most 32 groups
// (a group per thread of a warp in the standalone kernel, a group per row of
// threads in the fused tail).

struct ReduceGroups {
    int64_t size;   // partial rows per group
    int count;      // groups, 1..kMaxReduceGroups
};

constexpr int kMaxReduceGroups = 32;

__host__ __device__ inline ReduceGroups reduce_groups(int64_t G)
{
    int64_t s = 1;
    while (s * s < G) ++s;                   // ceil(sqrt(G)); G <= 2^31, a host-side call
    const int64_t s32 = (G + kMaxReduceGroups - 1) / kMaxReduceGroups;
    if (s32 > s) s = s32;
    ReduceGroups g;
    g.size = s;
    g.count = (int)((G + s - 1) / s);
    return g;
}

// dwh, dwe of the four columns 4f..4f+3 from their sums P.
__device__ __forceinline__ void write_weight_grads(int f, float4 P, const __nv_bfloat16 *wh,
                                                   const __nv_bfloat16 *we, float *dwh, float *dwe)
{
    const float p[4] = {P.x, P.y, P.z, P.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const int j = 4 * f + e;
        dwh[j] = __bfloat162float(we[j]) * p[e];
        dwe[j] = __bfloat162float(wh[j]) * p[e];
    }
}

// Level two fused into the tail of the backward kernel, instead of a second
// launch.  Every CTA writes its partial row, then takes a ticket: tickets[0]
// counts the CTAs that have.  The last K CTAs to take one (K slices of the
// columns; at most G, and at most `kmax`, half the CTAs the GPU holds at once)
// each wait, with a time limit, until all G have, and then reduce one slice
// of the columns over all G rows in the order above; the other CTAs exit.
// The CTAs that wait are the last ones to finish their tokens, so their SMs
// have nothing else to do, and they never hold all the SM slots, so every CTA
// still to come can be scheduled.  Within a slice, thread (q, c) sums the
// rows of group q for float4 column c in row order, and the group sums are
// added in group order through shared memory (`red`, blockDim.x float4).
// tickets[1] counts the slices done; the CTA that completes the last one sets
// both counters back to zero for the next call.  `flag` is one word of shared
// memory.  A wait that runs out of time records the pipeline-timeout code.
__device__ __forceinline__ void grad_w_reduce_tail(const float *w_partial, int64_t G, int H,
                                                   ReduceGroups grp, int kmax, unsigned int *tickets,
                                                   const __nv_bfloat16 *wh, const __nv_bfloat16 *we,
                                                   float *dwh, float *dwe, unsigned int *flag,
                                                   float4 *red)
{
    const int nt = blockDim.x, tid = threadIdx.x;
    const int nf4 = H >> 2;
    const int F = nt / grp.count;                       // float4 columns at a time (count <= 32 <= nt)
    int64_t K = (nf4 + F - 1) / F;
    if (K > G) K = G;
    if (K > kmax) K = kmax;
    const int Fk = (int)((nf4 + K - 1) / K);            // float4 columns per slice
    __threadfence();                                    // the partial row, before the ticket
    __syncthreads();
    if (tid == 0) *flag = atomicAdd(&tickets[0], 1u);
    __syncthreads();
    const int64_t t = *flag;
    if (t < G - K) return;
    const int64_t slice = t - (G - K);
    if (tid == 0) {
        const volatile unsigned int *arrived = tickets;
        const uint64_t t0 = globaltimer_ns();
        while (*arrived < (unsigned int)G) {
            if (globaltimer_ns() - t0 > kWaitLimitNs) {
                record_device_error(kErrPipelineTimeout);
                break;
            }
            __nanosleep(128);
        }
    }
    __syncthreads();
    __threadfence();                                    // every partial row, after the last ticket
    const int q = tid / F, c = tid % F;
    const int64_t r0 = (int64_t)q * grp.size;
    const int64_t r1 = (q < grp.count) ? ((G - r0 < grp.size) ? G : r0 + grp.size) : r0;
    const int fs = (int)(slice * Fk);
    const int fe = (fs + Fk < nf4) ? fs + Fk : nf4;
    for (int f0 = fs; f0 < fe; f0 += F) {
        const int f = f0 + c;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        if (q < grp.count && f < fe) {
            const float4 *col = reinterpret_cast<const float4 *>(w_partial) + f;
            for (int64_t r = r0; r < r1; r += 8) {
                float4 v[8];
#pragma unroll
                for (int u = 0; u < 8; ++u)
                    if (r + u < r1) v[u] = __ldcg(col + (r + u) * nf4);
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    if (r + u < r1) {
                        acc.x += v[u].x;
                        acc.y += v[u].y;
                        acc.z += v[u].z;
                        acc.w += v[u].w;
                    }
                }
            }
        }
        if (q < grp.count) red[q * F + c] = acc;
        __syncthreads();
        if (q == 0 && f < fe) {
            float4 P = make_float4(0.f, 0.f, 0.f, 0.f);
            for (int g = 0; g < grp.count; ++g) {
                const float4 rg = red[g * F + c];
                P.x += rg.x;
                P.y += rg.y;
                P.z += rg.z;
                P.w += rg.w;
            }
            write_weight_grads(f, P, wh, we, dwh, dwe);
        }
        __syncthreads();
    }
    if (tid == 0 && atomicAdd(&tickets[1], 1u) == (unsigned int)(K - 1)) {
        tickets[0] = 0u;
        tickets[1] = 0u;
    }
}

// -------------------------------------------------------------- backward ----

// Backward kernel with MAXV vectors per thread and at most MAXT threads per
// CTA.  The launch bound sets the register budget: at MAXV = 2 a CTA of up to
// 448 threads (rows of up to 7168 values) may hold 144 registers per thread,
// room for the fused weight in fp64 as well as fp32 (pass 1 then converts
// only x·k to fp64, not w); the 512-thread variant covers rows up to 8192.
template <int MAXV, int MAXT = gate_max_threads(MAXV), bool FUSED = false>
__global__ void __launch_bounds__(MAXT, 1)
gate_bwd_kernel(const uint4 *__restrict__ gout, const uint4 *__restrict__ x,
                const uint4 *__restrict__ k, const uint4 *__restrict__ v,
                const uint4 *__restrict__ wh, const uint4 *__restrict__ we, int64_t T, int H,
                float eps, float scalar, uint4 *__restrict__ dx, uint4 *__restrict__ dk,
                uint4 *__restrict__ dv, float *w_partial, int nstage,
                unsigned int *tickets, ReduceGroups grp, int kmax, float *dwh, float *dwe)
{
    extern __shared__ __align__(128) unsigned char smem[];
    const int nvec = H >> 3;
    const uint32_t row_bytes = (uint32_t)H * 2u;
    const uint32_t stage_bytes = 4u * row_bytes;
    unsigned char *tail = smem + (size_t)nstage * stage_bytes;
    float4 *red = reinterpret_cast<float4 *>(tail);                              // [2][32]
    double *redd = reinterpret_cast<double *>(tail + 2 * 32 * sizeof(float4));   // [2][32]
    const uint32_t bar0 = smem_addr(tail + kGateRedBytes);

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int nthreads = blockDim.x, nwarps = nthreads >> 5;

    float2 w[MAXV][4], acc[MAXV][4];
#pragma unroll
    for (int m = 0; m < MAXV; ++m) {
        const int vi = tid + m * nthreads;
        if (vi < nvec) {
            float2 a[4], b[4];
            unpack4x2(wh[vi], a);
            unpack4x2(we[vi], b);
#pragma unroll
            for (int e = 0; e < 4; ++e) w[m][e] = __fmul2_rn(a[e], b[e]);
        } else {
#pragma unroll
            for (int e = 0; e < 4; ++e) w[m][e] = make_float2(0.f, 0.f);
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[m][e] = make_float2(0.f, 0.f);
    }

    // the fused weight in fp64 for the dot product (exact: w is an fp32 value)
    double wd[MAXV][8];
#pragma unroll
    for (int m = 0; m < MAXV; ++m) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            wd[m][2 * e] = (double)w[m][e].x;
            wd[m][2 * e + 1] = (double)w[m][e].y;
        }
    }

    const int64_t G = gridDim.x, first = blockIdx.x;
    const int64_t nrows = T > first ? (T - first + G - 1) / G : 0;
    const void *src[4] = {gout, x, k, v};
    gate_pipeline_start<4>(smem, bar0, src, first, G, nrows, row_bytes, nstage);

    const float inv_h = 1.0f / (float)H;
    for (int64_t i = 0; i < nrows; ++i) {
        const int s = (int)(i % nstage);
        const bool ok = mbar_wait_bounded(bar0 + 8u * s, (uint32_t)((i / nstage) & 1));
        const uint4 *sg = reinterpret_cast<const uint4 *>(smem + (size_t)s * stage_bytes);
        const uint4 *sx = sg + nvec;
        const uint4 *sk = sx + nvec;
        const uint4 *sv = sk + nvec;

        uint4 gq[MAXV], xq[MAXV], kq[MAXV];
        float2 px2 = make_float2(0.f, 0.f), pk2 = px2, pg2 = px2;
        double pa = 0.0;
#pragma unroll
        for (int m = 0; m < MAXV; ++m) {
            const int vi = tid + m * nthreads;
            if (vi < nvec) {
                gq[m] = sg[vi];
                xq[m] = sx[vi];
                kq[m] = sk[vi];
                float2 gf[4], xf[4], kf[4], vf[4];
                unpack4x2(gq[m], gf);
                unpack4x2(xq[m], xf);
                unpack4x2(kq[m], kf);
                unpack4x2(sv[vi], vf);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    px2 = __ffma2_rn(xf[e], xf[e], px2);
                    pk2 = __ffma2_rn(kf[e], kf[e], pk2);
                    pg2 = __ffma2_rn(gf[e], vf[e], pg2);
                    const float2 xk = __fmul2_rn(xf[e], kf[e]);   // exact
                    pa = fma((double)xk.x, wd[m][2 * e], pa);
                    pa = fma((double)xk.y, wd[m][2 * e + 1], pa);
                }
            }
        }
        float px = warp_sum(px2.x + px2.y);
        float pk = warp_sum(pk2.x + pk2.y);
        float pg = warp_sum(pg2.x + pg2.y);
        pa = warp_sum_f64(pa);
        float4 *rb = red + (i & 1) * 32;
        double *rbd = redd + (i & 1) * 32;
        if (lane == 0) {
            rb[warp] = make_float4(px, pk, pg, 0.f);
            rbd[warp] = pa;
        }
        if (__syncthreads_or(!ok)) {
            // (with the fused reduction the CTA then takes no ticket: the
            // CTAs waiting in the tail give up at their own time limit)
            if (tid == 0) {
                record_device_error(kErrPipelineTimeout);
                gate_drain(bar0, i, nrows, nstage);
            }
            return;
        }
        if (tid == 0 && i + nstage < nrows)
            gate_issue_row<4>(smem, bar0, src, first + (i + nstage) * G, row_bytes, s);

        float4 r;
        double A;
        combine_partials(rb, rbd, nwarps, r, A);
        const float Sg = r.z;
        const GateScalars c = gate_scalars(r.x, r.y, A, inv_h, eps, scalar);
        // chain rule through sigmoid, signed_sqrt (|s| clamped at 1e-6), scalar
        const float du = Sg * c.gate * (1.0f - c.gate);
        const float dd = du * 0.5f * rsqrtf(fmaxf(fabsf(c.s), 1e-6f)) * scalar;
        const float c1 = dd * c.rx * c.rk;                // coefficient of w_j k_j in dx, w_j x_j in dk
        const float c2 = dd * c.d * c.rx * c.rx * inv_h;  // RMS term of x
        const float c3 = dd * c.d * c.rk * c.rk * inv_h;  // RMS term of k

        const int64_t row = first + i * G;
        uint4 *dxr = dx + row * nvec;
        uint4 *dkr = dk + row * nvec;
        uint4 *dvr = dv + row * nvec;
        const float2 c1v = make_float2(c1, c1), nc2 = make_float2(-c2, -c2);
        const float2 nc3 = make_float2(-c3, -c3), gate2 = make_float2(c.gate, c.gate);
#pragma unroll
        for (int m = 0; m < MAXV; ++m) {
            const int vi = tid + m * nthreads;
            if (vi < nvec) {
                float2 gf[4], xf[4], kf[4], a[4], b[4], cv[4];
                unpack4x2(gq[m], gf);
                unpack4x2(xq[m], xf);
                unpack4x2(kq[m], kf);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 cw = __fmul2_rn(c1v, w[m][e]);
                    a[e] = __ffma2_rn(nc2, xf[e], __ffma2_rn(cw, kf[e], gf[e]));
                    b[e] = __ffma2_rn(nc3, kf[e], __fmul2_rn(cw, xf[e]));
                    cv[e] = __fmul2_rn(gate2, gf[e]);
                    acc[m][e] = __ffma2_rn(c1v, __fmul2_rn(xf[e], kf[e]), acc[m][e]);
                }
                __stcs(dxr + vi, pack4x2(a));
                __stcs(dkr + vi, pack4x2(b));
                __stcs(dvr + vi, pack4x2(cv));
            }
        }
    }

    // The weight-gradient reduction launched after this kernel may now be
    // scheduled (it waits for this whole grid before it reads the partials).
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    // Level one of the weight-gradient reduction: this CTA's partial row.
    float4 *prow = reinterpret_cast<float4 *>(w_partial + (int64_t)blockIdx.x * H);
#pragma unroll
    for (int m = 0; m < MAXV; ++m) {
        const int vi = tid + m * nthreads;
        if (vi < nvec) {
            prow[2 * vi] = make_float4(acc[m][0].x, acc[m][0].y, acc[m][1].x, acc[m][1].y);
            prow[2 * vi + 1] = make_float4(acc[m][2].x, acc[m][2].y, acc[m][3].x, acc[m][3].y);
        }
    }
    // (the data stages are idle now: their shared memory holds the tail's
    // group sums, at most blockDim.x float4, which fit in two stages)
    if (FUSED)
        grad_w_reduce_tail(w_partial, G, H, grp, kmax, tickets, reinterpret_cast<const __nv_bfloat16 *>(wh),
                           reinterpret_cast<const __nv_bfloat16 *>(we), dwh, dwe,
                           reinterpret_cast<unsigned int *>(red), reinterpret_cast<float4 *>(smem));
}

// ------------------------------------------ standalone weight-gradient level 2 ----

constexpr int kReduceThreads = 1024;
constexpr int kReduceWarps = kReduceThreads / 32;
static_assert(kReduceWarps >= kMaxReduceGroups, "one warp per group");

// Standalone level two, in the order above: per block of 32 columns, warp q
// sums the rows of group q in order, then warp 0 adds the group sums in group
// order.
__global__ void __launch_bounds__(kReduceThreads)
grad_w_reduce_kernel(const float *__restrict__ w_partial, int64_t G, ReduceGroups grp, int H,
                     const __nv_bfloat16 *__restrict__ wh, const __nv_bfloat16 *__restrict__ we,
                     float *__restrict__ dwh, float *__restrict__ dwe)
{
    __shared__ float part[kReduceWarps][33];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    // launched with programmatic stream serialisation: wait for the backward
    // kernel that wrote the partials (a no-op after any other predecessor)
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int col = blockIdx.x * 32 + lane;
    float a = 0.f;
    if (col < H && warp < grp.count) {
        const float *p = w_partial + col;
        const int64_t p0 = (int64_t)warp * grp.size;
        const int64_t p1 = (G - p0 < grp.size) ? G : p0 + grp.size;
        int64_t r = p0;
        for (; r + 3 < p1; r += 4) {
            const float v0 = p[r * H], v1 = p[(r + 1) * H], v2 = p[(r + 2) * H], v3 = p[(r + 3) * H];
            a += v0;
            a += v1;
            a += v2;
            a += v3;
        }
        for (; r < p1; ++r) a += p[r * H];
    }
    part[warp][lane] = a;
    __syncthreads();
    if (warp == 0 && col < H) {
        float P = 0.f;
        for (int q = 0; q < grp.count; ++q) P += part[q][lane];
        dwh[col] = __bfloat162float(we[col]) * P;
        dwe[col] = __bfloat162float(wh[col]) * P;
    }
}

}  // namespace engram
