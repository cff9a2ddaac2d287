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

// Largest CTA of a gate kernel whose threads own MAXV column vectors each.
template <int MAXV>
constexpr int gate_max_threads() { return 1024 / MAXV; }
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
    mbar_arrive_expect_tx(bar, stage_bytes);
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
__global__ void __launch_bounds__(gate_max_threads<MAXV>(), MAXV == 4 ? 2 : 1)
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
        float a[8], b[8];
        if (vi < nvec) {
            unpack8(wh[vi], a);
            unpack8(we[vi], b);
        } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) a[e] = b[e] = 0.f;
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) w[m][e] = (double)(a[e] * b[e]);
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
        float px = 0.f, pk = 0.f;
        double pa = 0.0;
#pragma unroll
        for (int m = 0; m < MAXV; ++m) {
            const int vi = tid + m * nthreads;
            if (vi < nvec) {
                xq[m] = sx[vi];
                vq[m] = sv[vi];
                float xf[8], kf[8];
                unpack8(xq[m], xf);
                unpack8(sk[vi], kf);
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    px = fmaf(xf[e], xf[e], px);
                    pk = fmaf(kf[e], kf[e], pk);
                    pa = fma((double)(xf[e] * kf[e]), w[m][e], pa);
                }
            }
        }
        px = warp_sum(px);
        pk = warp_sum(pk);
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

        float Sx = 0.f, Sk = 0.f;
        double A = 0.0;
        for (int q = 0; q < nwarps; ++q) {
            const float4 r = rb[q];
            Sx += r.x;
            Sk += r.y;
            A += rbd[q];
        }
        const GateScalars c = gate_scalars(Sx, Sk, A, inv_h, eps, scalar);

        const int64_t row = first + i * G;
        uint4 *orow = out + row * nvec;
#pragma unroll
        for (int m = 0; m < MAXV; ++m) {
            const int vi = tid + m * nthreads;
            if (vi < nvec) {
                float xf[8], vf[8], of[8];
                unpack8(xq[m], xf);
                unpack8(vq[m], vf);
#pragma unroll
                for (int e = 0; e < 8; ++e) of[e] = fmaf(c.gate, vf[e], xf[e]);
                __stcs(orow + vi, pack8(of));
            }
        }
        if (tid == 0 && gate != nullptr) gate[row] = c.gate;
    }
}

// -------------------------------------------------------------- backward ----

template <int MAXV>
__global__ void __launch_bounds__(gate_max_threads<MAXV>(), 1)
gate_bwd_kernel(const uint4 *__restrict__ gout, const uint4 *__restrict__ x,
                const uint4 *__restrict__ k, const uint4 *__restrict__ v,
                const uint4 *__restrict__ wh, const uint4 *__restrict__ we, int64_t T, int H,
                float eps, float scalar, uint4 *__restrict__ dx, uint4 *__restrict__ dk,
                uint4 *__restrict__ dv, float *__restrict__ w_partial, int nstage)
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

    float w[MAXV][8], acc[MAXV][8];
#pragma unroll
    for (int m = 0; m < MAXV; ++m) {
        const int vi = tid + m * nthreads;
        if (vi < nvec) {
            float a[8], b[8];
            unpack8(wh[vi], a);
            unpack8(we[vi], b);
#pragma unroll
            for (int e = 0; e < 8; ++e) w[m][e] = a[e] * b[e];
        } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) w[m][e] = 0.f;
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[m][e] = 0.f;
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
        float px = 0.f, pk = 0.f, pg = 0.f;
        double pa = 0.0;
#pragma unroll
        for (int m = 0; m < MAXV; ++m) {
            const int vi = tid + m * nthreads;
            if (vi < nvec) {
                gq[m] = sg[vi];
                xq[m] = sx[vi];
                kq[m] = sk[vi];
                float gf[8], xf[8], kf[8], vf[8];
                unpack8(gq[m], gf);
                unpack8(xq[m], xf);
                unpack8(kq[m], kf);
                unpack8(sv[vi], vf);
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    px = fmaf(xf[e], xf[e], px);
                    pk = fmaf(kf[e], kf[e], pk);
                    pa = fma((double)(xf[e] * kf[e]), (double)w[m][e], pa);
                    pg = fmaf(gf[e], vf[e], pg);
                }
            }
        }
        px = warp_sum(px);
        pk = warp_sum(pk);
        pa = warp_sum_f64(pa);
        pg = warp_sum(pg);
        float4 *rb = red + (i & 1) * 32;
        double *rbd = redd + (i & 1) * 32;
        if (lane == 0) {
            rb[warp] = make_float4(px, pk, pg, 0.f);
            rbd[warp] = pa;
        }
        if (__syncthreads_or(!ok)) {
            if (tid == 0) {
                record_device_error(kErrPipelineTimeout);
                gate_drain(bar0, i, nrows, nstage);
            }
            return;
        }
        if (tid == 0 && i + nstage < nrows)
            gate_issue_row<4>(smem, bar0, src, first + (i + nstage) * G, row_bytes, s);

        float Sx = 0.f, Sk = 0.f, Sg = 0.f;
        double A = 0.0;
        for (int q = 0; q < nwarps; ++q) {
            const float4 r = rb[q];
            Sx += r.x;
            Sk += r.y;
            Sg += r.z;
            A += rbd[q];
        }
        const GateScalars c = gate_scalars(Sx, Sk, A, inv_h, eps, scalar);
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
#pragma unroll
        for (int m = 0; m < MAXV; ++m) {
            const int vi = tid + m * nthreads;
            if (vi < nvec) {
                float gf[8], xf[8], kf[8], a[8], b[8], cv[8];
                unpack8(gq[m], gf);
                unpack8(xq[m], xf);
                unpack8(kq[m], kf);
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const float cw = c1 * w[m][e];
                    a[e] = fmaf(-c2, xf[e], fmaf(cw, kf[e], gf[e]));
                    b[e] = fmaf(-c3, kf[e], cw * xf[e]);
                    cv[e] = c.gate * gf[e];
                    acc[m][e] = fmaf(c1, xf[e] * kf[e], acc[m][e]);
                }
                __stcs(dxr + vi, pack8(a));
                __stcs(dkr + vi, pack8(b));
                __stcs(dvr + vi, pack8(cv));
            }
        }
    }

    // Level one of the weight-gradient reduction: this CTA's partial row.
    float4 *prow = reinterpret_cast<float4 *>(w_partial + (int64_t)blockIdx.x * H);
#pragma unroll
    for (int m = 0; m < MAXV; ++m) {
        const int vi = tid + m * nthreads;
        if (vi < nvec) {
            prow[2 * vi] = make_float4(acc[m][0], acc[m][1], acc[m][2], acc[m][3]);
            prow[2 * vi + 1] = make_float4(acc[m][4], acc[m][5], acc[m][6], acc[m][7]);
        }
    }
}

// ------------------------------------------------ weight-gradient level 2 ----

constexpr int kReduceThreads = 1024;
constexpr int kReduceWarps = kReduceThreads / 32;

// P_j = sum_{p<G} w_partial[p][j] for the 32 columns of a block: warp q sums
// partial rows p = q, q + 32, q + 64, ... in order, then warp 0 adds the 32
// warp sums in warp order, so the result depends only on G.  dwh = we * P,
// dwe = wh * P.
__global__ void __launch_bounds__(kReduceThreads)
grad_w_reduce_kernel(const float *__restrict__ w_partial, int64_t G, int H,
                     const __nv_bfloat16 *__restrict__ wh, const __nv_bfloat16 *__restrict__ we,
                     float *__restrict__ dwh, float *__restrict__ dwe)
{
    __shared__ float part[kReduceWarps][33];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int col = blockIdx.x * 32 + lane;
    float a = 0.f;
    if (col < H) {
        const float *p = w_partial + col;
        int64_t q = warp;
        for (; q + 3 * kReduceWarps < G; q += 4 * kReduceWarps) {
            const float v0 = p[q * H], v1 = p[(q + kReduceWarps) * H],
                        v2 = p[(q + 2 * kReduceWarps) * H], v3 = p[(q + 3 * kReduceWarps) * H];
            a += v0;
            a += v1;
            a += v2;
            a += v3;
        }
        for (; q < G; q += kReduceWarps) a += p[q * H];
    }
    part[warp][lane] = a;
    __syncthreads();
    if (warp == 0 && col < H) {
        float P = 0.f;
#pragma unroll
        for (int q = 0; q < kReduceWarps; ++q) P += part[q][lane];
        dwh[col] = __bfloat162float(we[col]) * P;
        dwe[col] = __bfloat162float(wh[col]) * P;
    }
}

}  // namespace engram
