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
// tokens ahead of the compute.  Each thread owns the same 16-byte column
// vectors j = tid + m * blockDim.x of every token, so the fused weight and the
// backward's weight-gradient accumulators stay in registers for the whole
// kernel.  Per token: one pass over the staged rows accumulates the fp32
// statistics (sum x^2, sum k^2, sum x k w, and sum g v for the backward) into
// registers, one warp-shuffle + shared-memory block reduction combines them in
// a fixed order, and the outputs are computed from the registers and stored
// with streaming (evict-first) 16-byte stores.  The stage is handed back to the
// copy engine right after the block reduction, since its contents already
// live in registers.
#pragma once

#include "common.cuh"

namespace engram {

// Largest CTA of the gate kernels; a thread owns at most MAXV column vectors.
constexpr int kGateMaxThreads = 512;
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

// Issue the bulk copies of token `row` (ntensors rows of row_bytes) into stage
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

// After a failed wait: wait (sharing one time limit) for every copy still in
// flight into this CTA's shared memory, so that none lands after the CTA exits.
__device__ __forceinline__ double warp_sum_f64(double v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

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

// --------------------------------------------------------------- forward ----

template <int MAXV>
__global__ void __launch_bounds__(kGateMaxThreads, 1)
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

    float w[MAXV][8];
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
    }

    const int64_t G = gridDim.x, first = blockIdx.x;
    const int64_t nrows = T > first ? (T - first + G - 1) / G : 0;
    const void *src[3] = {x, k, v};

    if (tid == 0) {
        for (int s = 0; s < nstage; ++s) mbar_init(bar0 + 8u * s, 1);
        fence_barrier_init();
    }
    __syncthreads();
    if (tid == 0) {
        const int64_t pre = nrows < nstage ? nrows : nstage;
        for (int64_t i = 0; i < pre; ++i)
            gate_issue_row<3>(smem, bar0, src, first + i * G, row_bytes, (int)(i % nstage));
    }

    const float fH = (float)H;
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
                    // x*k is exact in fp32; the dot product is summed in fp64
                    pa = fma((double)(xf[e] * kf[e]), (double)w[m][e], pa);
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
        double Ad = 0.0;
        for (int q = 0; q < nwarps; ++q) {
            const float4 r = rb[q];
            Sx += r.x;
            Sk += r.y;
            Ad += rbd[q];
        }
        const float A = (float)Ad;
        const float rx = 1.0f / sqrtf(Sx / fH + eps);
        const float rk = 1.0f / sqrtf(Sk / fH + eps);
        const float sarg = (rx * rk * A) * scalar;
        const float u = copysignf(sqrtf(fabsf(sarg)), sarg);
        const float g = 1.0f / (1.0f + expf(-u));

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
                for (int e = 0; e < 8; ++e) of[e] = fmaf(g, vf[e], xf[e]);
                __stcs(orow + vi, pack8(of));
            }
        }
        if (tid == 0 && gate != nullptr) gate[row] = g;
    }
}

// -------------------------------------------------------------- backward ----

template <int MAXV>
__global__ void __launch_bounds__(kGateMaxThreads, 1)
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

    if (tid == 0) {
        for (int s = 0; s < nstage; ++s) mbar_init(bar0 + 8u * s, 1);
        fence_barrier_init();
    }
    __syncthreads();
    if (tid == 0) {
        const int64_t pre = nrows < nstage ? nrows : nstage;
        for (int64_t i = 0; i < pre; ++i)
            gate_issue_row<4>(smem, bar0, src, first + i * G, row_bytes, (int)(i % nstage));
    }

    const float fH = (float)H;
    for (int64_t i = 0; i < nrows; ++i) {
        const int s = (int)(i % nstage);
        const bool ok = mbar_wait_bounded(bar0 + 8u * s, (uint32_t)((i / nstage) & 1));
        const uint4 *sg = reinterpret_cast<const uint4 *>(smem + (size_t)s * stage_bytes);
        const uint4 *sx = sg + nvec;
        const uint4 *sk = sx + nvec;
        const uint4 *sv = sk + nvec;

        uint4 gq[MAXV], xq[MAXV], kq[MAXV], vq[MAXV];
        float px = 0.f, pk = 0.f, pg = 0.f;
        double pa = 0.0;
#pragma unroll
        for (int m = 0; m < MAXV; ++m) {
            const int vi = tid + m * nthreads;
            if (vi < nvec) {
                gq[m] = sg[vi];
                xq[m] = sx[vi];
                kq[m] = sk[vi];
                vq[m] = sv[vi];
                float gf[8], xf[8], kf[8], vf[8];
                unpack8(gq[m], gf);
                unpack8(xq[m], xf);
                unpack8(kq[m], kf);
                unpack8(vq[m], vf);
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
        double Ad = 0.0;
        for (int q = 0; q < nwarps; ++q) {
            const float4 r = rb[q];
            Sx += r.x;
            Sk += r.y;
            Sg += r.z;
            Ad += rbd[q];
        }
        const float A = (float)Ad;
        const float rx = 1.0f / sqrtf(Sx / fH + eps);
        const float rk = 1.0f / sqrtf(Sk / fH + eps);
        const float d = rx * rk * A;
        const float sarg = d * scalar;
        const float u = copysignf(sqrtf(fabsf(sarg)), sarg);
        const float gate = 1.0f / (1.0f + expf(-u));
        // chain rule through sigmoid, signed_sqrt (|s| clamped at 1e-6), scalar
        const float du = Sg * gate * (1.0f - gate);
        const float dd = du / (2.0f * sqrtf(fmaxf(fabsf(sarg), 1e-6f))) * scalar;
        const float c1 = dd * rx * rk;            // d dot / d(x_j k_j w_j) * dd
        const float c2 = dd * d * rx * rx / fH;   // RMS term of x
        const float c3 = dd * d * rk * rk / fH;   // RMS term of k

        const int64_t row = first + i * G;
        uint4 *dxr = dx + row * nvec;
        uint4 *dkr = dk + row * nvec;
        uint4 *dvr = dv + row * nvec;
#pragma unroll
        for (int m = 0; m < MAXV; ++m) {
            const int vi = tid + m * nthreads;
            if (vi < nvec) {
                float gf[8], xf[8], kf[8], a[8], b[8], c[8];
                unpack8(gq[m], gf);
                unpack8(xq[m], xf);
                unpack8(kq[m], kf);
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const float cw = c1 * w[m][e];
                    a[e] = fmaf(-c2, xf[e], fmaf(cw, kf[e], gf[e]));
                    b[e] = fmaf(-c3, kf[e], cw * xf[e]);
                    c[e] = gate * gf[e];
                    acc[m][e] = fmaf(c1, xf[e] * kf[e], acc[m][e]);
                }
                __stcs(dxr + vi, pack8(a));
                __stcs(dkr + vi, pack8(b));
                __stcs(dvr + vi, pack8(c));
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

// P_j = sum_{p<G} w_partial[p][j]: warp q of a block sums partial rows
// p = q, q+8, q+16, ... of its 32 columns in order, then warp 0 adds the 8
// warp sums in order; dwh = we * P, dwe = wh * P.
__global__ void __launch_bounds__(256)
grad_w_reduce_kernel(const float *__restrict__ w_partial, int64_t G, int H,
                     const __nv_bfloat16 *__restrict__ wh, const __nv_bfloat16 *__restrict__ we,
                     float *__restrict__ dwh, float *__restrict__ dwe)
{
    __shared__ float part[8][33];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int col = blockIdx.x * 32 + lane;
    float a = 0.f;
    if (col < H) {
        const float *p = w_partial + col;
        int64_t q = warp;
        for (; q + 24 < G; q += 32) {
            const float v0 = p[q * H], v1 = p[(q + 8) * H], v2 = p[(q + 16) * H],
                        v3 = p[(q + 24) * H];
            a += v0;
            a += v1;
            a += v2;
            a += v3;
        }
        for (; q < G; q += 8) a += p[q * H];
    }
    part[warp][lane] = a;
    __syncthreads();
    if (warp == 0 && col < H) {
        float P = 0.f;
#pragma unroll
        for (int q = 0; q < 8; ++q) P += part[q][lane];
        dwh[col] = __bfloat162float(we[col]) * P;
        dwe[col] = __bfloat162float(wh[col]) * P;
    }
}

}  // namespace engram
