// Engram gate for any hidden size (sm_100a).
//
// The same forward and backward as gate_kernels.cuh (the gate of the page
// "DeepSeek 开源 TileKernels", zhichai.net/topic/177618722, section
// "5. Engram — 条件记忆门控"), for the shapes the tuned kernels do not take:
// H not a multiple of 8, H above 8192, or bf16 tensors that do not start on a
// 16-byte boundary (their rows cannot be moved with 16-byte bulk copies).
//
// One CTA per token at a time (persistent: CTA c handles tokens c, c+G, ...;
// gen_threads(H) threads, 64 to 256), two passes over the token's rows,
// consecutive threads on consecutive columns: the first pass accumulates the
// statistics (fp32 sums of squares and of
// g*v, the dot product sum x k w in fp64 exactly as the tuned kernels do), a
// fixed-order block reduction combines them, the per-token scalars come from
// the same gate_scalars(), and the second pass reads the rows again (from L2:
// a token's rows were just read) to write the outputs.
//
// VEC: every token tensor (inputs and outputs) starts at the same offset from
// a 16-byte boundary, so in every row the same columns fall on 16-byte
// boundaries.  A row is then split into a head (the columns before the first
// boundary, at most 7), a body of 16-byte vectors (8 columns, one vector per
// thread at a time) and a tail; head and tail are read element by element.
// Without VEC every column is read on its own.  The fused weight w = wh * we
// (4H bytes for the whole kernel, served by L1) is read 8 columns at a time;
// SHIFT (rows whose body vectors are not on 16-byte boundaries of wh and we:
// odd H, or tensors past a 16-byte boundary) reads it from the two aligned
// 16-byte chunks that cover each vector (wvec_at) instead of column by column.
// (The kernel without SHIFT is kept apart: the extra code, never run when
// every row is aligned, made the aligned case slower.)
//
// The backward adds c * x_j * k_j into the CTA's partial row (row c of
// w_partial belongs to CTA c alone and is updated in token order, so it is
// deterministic), kept in shared memory when H <= kGenSmemPartial.
#pragma once

#include "common.cuh"
#include "gate_kernels.cuh"

namespace engram {

constexpr int kGenThreads = 256;                 // the most threads a generic CTA has
constexpr int kGenWarps = kGenThreads / 32;

// Threads of a generic CTA for rows of H values: enough for one 16-byte vector
// (8 values) per thread, between 64 and 256, so that short rows keep more
// tokens in flight per SM instead of idle threads.
__host__ __device__ constexpr int gen_threads(int H)
{
    return (H + 7) / 8 + 1 <= 64 ? 64 : (H + 7) / 8 + 1 <= 128 ? 128 : 256;
}
constexpr int kGenMaxH = 65536;
constexpr int kGenSmemPartial = 24576;   // partial row in shared memory up to this H (96 KB)

__device__ __forceinline__ float bf(const __nv_bfloat16 *p) { return __bfloat162float(*p); }

__device__ __forceinline__ float wcol(const __nv_bfloat16 *wh, const __nv_bfloat16 *we, int j)
{
    return bf(wh + j) * bf(we + j);   // exact in fp32
}

// The fused weight of the 8 columns j..j+7: one 16-byte load of wh and of we
// when both are on a 16-byte boundary there, else column by column.
__device__ __forceinline__ void wvec(const __nv_bfloat16 *wh, const __nv_bfloat16 *we, int j, float w[8])
{
    if (((reinterpret_cast<uintptr_t>(wh + j) | reinterpret_cast<uintptr_t>(we + j)) & 15u) == 0) {
        float2 a[4], b[4];
        unpack4x2(*reinterpret_cast<const uint4 *>(wh + j), a);
        unpack4x2(*reinterpret_cast<const uint4 *>(we + j), b);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            w[2 * e] = a[e].x * b[e].x;
            w[2 * e + 1] = a[e].y * b[e].y;
        }
    } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) w[e] = wcol(wh, we, j + e);
    }
}

// Lanes h..h+7 of the 16 bf16 lanes of (lo, hi): the 8 values of a vector
// that starts h values past a 16-byte boundary, from the two aligned 16-byte
// chunks that hold it.
template <int h>
__device__ __forceinline__ uint4 lanes_from(const uint4 &lo, const uint4 &hi)
{
    const uint32_t a[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
    uint32_t o[4];
#pragma unroll
    for (int k = 0; k < 4; ++k)
        o[k] = (h & 1) ? __funnelshift_r(a[h / 2 + k], a[h / 2 + k + 1], 16) : a[h / 2 + k];
    return make_uint4(o[0], o[1], o[2], o[3]);
}

__device__ __forceinline__ uint4 lanes_from(const uint4 &lo, const uint4 &hi, int h)
{
    switch (h) {
    case 1: return lanes_from<1>(lo, hi);
    case 2: return lanes_from<2>(lo, hi);
    case 3: return lanes_from<3>(lo, hi);
    case 4: return lanes_from<4>(lo, hi);
    case 5: return lanes_from<5>(lo, hi);
    case 6: return lanes_from<6>(lo, hi);
    case 7: return lanes_from<7>(lo, hi);
    default: return lo;
    }
}

// The fused weight of the 8 columns j..j+7 of a body vector whose row starts
// h = j % 8 values past a 16-byte boundary (h uniform over the CTA for one
// row): where wh and we are 16-byte aligned, from the two aligned 16-byte
// chunks of each that cover the columns (4 loads instead of 16), as long as
// the second chunk lies inside the arrays; else as wvec.
__device__ __forceinline__ void wvec_at(const __nv_bfloat16 *wh, const __nv_bfloat16 *we, int j, int H,
                                        bool w_aligned, float w[8])
{
    const int h = j & 7;
    if (h == 0 || !w_aligned || j - h + 16 > H) {
        wvec(wh, we, j, w);
        return;
    }
    const uint4 *a = reinterpret_cast<const uint4 *>(wh + (j - h));
    const uint4 *b = reinterpret_cast<const uint4 *>(we + (j - h));
    float2 fa[4], fb[4];
    unpack4x2(lanes_from(a[0], a[1], h), fa);
    unpack4x2(lanes_from(b[0], b[1], h), fb);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        w[2 * e] = fa[e].x * fb[e].x;
        w[2 * e + 1] = fa[e].y * fb[e].y;
    }
}

// Columns of a row before its first 16-byte boundary (0..7, at most H).
__device__ __forceinline__ int row_head(const void *row, int H)
{
    const int past = (int)((reinterpret_cast<uintptr_t>(row) >> 1) & 7u);   // bf16 past a boundary
    const int head = (8 - past) & 7;
    return head < H ? head : H;
}

// Block sums of one token's statistics in a fixed order (warp shuffles, then
// the warps' partials in warp order).  Every thread gets the totals.
template <int NT>
__device__ __forceinline__ void gen_block_reduce(float px, float pk, float pg, double pa,
                                                 float4 *red, double *redd, float4 &r, double &A)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    px = warp_sum(px);
    pk = warp_sum(pk);
    pg = warp_sum(pg);
    pa = warp_sum_f64(pa);
    if (lane == 0) {
        red[warp] = make_float4(px, pk, pg, 0.f);
        redd[warp] = pa;
    }
    __syncthreads();
    r = make_float4(0.f, 0.f, 0.f, 0.f);
    A = 0.0;
#pragma unroll
    for (int w = 0; w < NT / 32; ++w) {
        const float4 t = red[w];
        r.x += t.x;
        r.y += t.y;
        r.z += t.z;
        A += redd[w];
    }
    __syncthreads();   // the buffers are reused by the next token
}

// Visit the columns of one row: f(j, false) for the single column j, or
// f(j, true) for the 8 columns j..j+7 of a 16-byte vector.  Thread tid takes
// head and tail column tid and body vectors tid, tid + NT, ... (NT threads)
template <bool VEC, int NT, typename F>
__device__ __forceinline__ void for_columns(const void *row, int H, F &&f)
{
    if (!VEC) {
        for (int j = threadIdx.x; j < H; j += NT) f(j, false);
        return;
    }
    const int head = row_head(row, H);
    const int nvec = (H - head) >> 3;
    const int tail = head + 8 * nvec;
    if ((int)threadIdx.x < head) f((int)threadIdx.x, false);
    for (int i = threadIdx.x; i < nvec; i += NT) f(head + 8 * i, true);
    if (tail + (int)threadIdx.x < H) f(tail + (int)threadIdx.x, false);
}

template <bool VEC, bool SHIFT, int NT>
__global__ void __launch_bounds__(NT)
gate_generic_fwd_kernel(const __nv_bfloat16 *__restrict__ x, const __nv_bfloat16 *__restrict__ k,
                        const __nv_bfloat16 *__restrict__ v, const __nv_bfloat16 *__restrict__ wh,
                        const __nv_bfloat16 *__restrict__ we, int64_t T, int H, float eps,
                        float scalar, __nv_bfloat16 *__restrict__ out, float *__restrict__ gate)
{
    __shared__ float4 red[kGenWarps];
    __shared__ double redd[kGenWarps];
    const float inv_h = 1.0f / (float)H;
    const bool w_aligned = ((reinterpret_cast<uintptr_t>(wh) | reinterpret_cast<uintptr_t>(we)) & 15u) == 0;
    for (int64_t t = blockIdx.x; t < T; t += gridDim.x) {
        const __nv_bfloat16 *xr = x + t * H, *kr = k + t * H, *vr = v + t * H;
        __nv_bfloat16 *orow = out + t * H;
        float px = 0.f, pk = 0.f;
        double pa = 0.0;
        for_columns<VEC, NT>(xr, H, [&](int j, bool vec) {
            if (vec) {
                float2 xf[4], kf[4];
                float w[8];
                unpack4x2(*reinterpret_cast<const uint4 *>(xr + j), xf);
                unpack4x2(*reinterpret_cast<const uint4 *>(kr + j), kf);
                if (SHIFT) wvec_at(wh, we, j, H, w_aligned, w);
                else wvec(wh, we, j, w);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    px = fmaf(xf[e].x, xf[e].x, fmaf(xf[e].y, xf[e].y, px));
                    pk = fmaf(kf[e].x, kf[e].x, fmaf(kf[e].y, kf[e].y, pk));
                    pa = fma((double)(xf[e].x * kf[e].x), (double)w[2 * e], pa);
                    pa = fma((double)(xf[e].y * kf[e].y), (double)w[2 * e + 1], pa);
                }
            } else {
                const float xv = bf(xr + j), kv = bf(kr + j);
                px = fmaf(xv, xv, px);
                pk = fmaf(kv, kv, pk);
                pa = fma((double)(xv * kv), (double)wcol(wh, we, j), pa);
            }
        });
        float4 r;
        double A;
        gen_block_reduce<NT>(px, pk, 0.f, pa, red, redd, r, A);
        const GateScalars c = gate_scalars(r.x, r.y, A, inv_h, eps, scalar);
        for_columns<VEC, NT>(xr, H, [&](int j, bool vec) {
            if (vec) {
                float2 xf[4], vf[4], of[4];
                unpack4x2(*reinterpret_cast<const uint4 *>(xr + j), xf);
                unpack4x2(*reinterpret_cast<const uint4 *>(vr + j), vf);
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    of[e] = make_float2(fmaf(c.gate, vf[e].x, xf[e].x), fmaf(c.gate, vf[e].y, xf[e].y));
                __stcs(reinterpret_cast<uint4 *>(orow + j), pack4x2(of));
            } else {
                orow[j] = __float2bfloat16_rn(fmaf(c.gate, bf(vr + j), bf(xr + j)));
            }
        });
        if (threadIdx.x == 0 && gate != nullptr) gate[t] = c.gate;
    }
}

template <bool VEC, bool SHIFT, int NT>
__global__ void __launch_bounds__(NT)
gate_generic_bwd_kernel(const __nv_bfloat16 *__restrict__ gout, const __nv_bfloat16 *__restrict__ x,
                        const __nv_bfloat16 *__restrict__ k, const __nv_bfloat16 *__restrict__ v,
                        const __nv_bfloat16 *__restrict__ wh, const __nv_bfloat16 *__restrict__ we,
                        int64_t T, int H, float eps, float scalar, __nv_bfloat16 *__restrict__ dx,
                        __nv_bfloat16 *__restrict__ dk, __nv_bfloat16 *__restrict__ dv,
                        float *__restrict__ w_partial)
{
    extern __shared__ __align__(16) float s_part[];   // H + 8 floats when H <= kGenSmemPartial
    __shared__ float4 red[kGenWarps];
    __shared__ double redd[kGenWarps];
    const float inv_h = 1.0f / (float)H;
    const bool w_aligned = ((reinterpret_cast<uintptr_t>(wh) | reinterpret_cast<uintptr_t>(we)) & 15u) == 0;
    float *prow = w_partial + (int64_t)blockIdx.x * H;
    // The partial row in shared memory starts `pad` floats in, chosen so that
    // the body vectors of this CTA's first token row (which start h columns
    // past a 16-byte boundary of the row) fall on 16-byte boundaries of the
    // array.  Every row of the CTA has that phase when G * H is a multiple of
    // 8 (odd H with the recommended G); rows of other phases take the
    // element-wise path below.
    const int pad = SHIFT ? (8 - row_head(x + (int64_t)blockIdx.x * H, H)) & 7 : 0;
    float *acc = H <= kGenSmemPartial ? s_part + pad : prow;
    for (int j = threadIdx.x; j < H; j += NT) acc[j] = 0.f;
    for (int64_t t = blockIdx.x; t < T; t += gridDim.x) {
        const __nv_bfloat16 *gr = gout + t * H, *xr = x + t * H, *kr = k + t * H, *vr = v + t * H;
        float px = 0.f, pk = 0.f, pg = 0.f;
        double pa = 0.0;
        for_columns<VEC, NT>(xr, H, [&](int j, bool vec) {
            if (vec) {
                float2 gf[4], xf[4], kf[4], vf[4];
                float w[8];
                unpack4x2(*reinterpret_cast<const uint4 *>(gr + j), gf);
                unpack4x2(*reinterpret_cast<const uint4 *>(xr + j), xf);
                unpack4x2(*reinterpret_cast<const uint4 *>(kr + j), kf);
                unpack4x2(*reinterpret_cast<const uint4 *>(vr + j), vf);
                if (SHIFT) wvec_at(wh, we, j, H, w_aligned, w);
                else wvec(wh, we, j, w);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    px = fmaf(xf[e].x, xf[e].x, fmaf(xf[e].y, xf[e].y, px));
                    pk = fmaf(kf[e].x, kf[e].x, fmaf(kf[e].y, kf[e].y, pk));
                    pg = fmaf(gf[e].x, vf[e].x, fmaf(gf[e].y, vf[e].y, pg));
                    pa = fma((double)(xf[e].x * kf[e].x), (double)w[2 * e], pa);
                    pa = fma((double)(xf[e].y * kf[e].y), (double)w[2 * e + 1], pa);
                }
            } else {
                const float xv = bf(xr + j), kv = bf(kr + j);
                px = fmaf(xv, xv, px);
                pk = fmaf(kv, kv, pk);
                pg = fmaf(bf(gr + j), bf(vr + j), pg);
                pa = fma((double)(xv * kv), (double)wcol(wh, we, j), pa);
            }
        });
        float4 r;
        double A;
        gen_block_reduce<NT>(px, pk, pg, pa, red, redd, r, A);
        const float Sg = r.z;
        const GateScalars c = gate_scalars(r.x, r.y, A, inv_h, eps, scalar);
        // chain rule through sigmoid, signed_sqrt (|s| clamped at 1e-6), scalar
        const float du = Sg * c.gate * (1.0f - c.gate);
        const float dd = du * 0.5f * rsqrtf(fmaxf(fabsf(c.s), 1e-6f)) * scalar;
        const float c1 = dd * c.rx * c.rk;
        const float c2 = dd * c.d * c.rx * c.rx * inv_h;
        const float c3 = dd * c.d * c.rk * c.rk * inv_h;
        __nv_bfloat16 *dxr = dx + t * H, *dkr = dk + t * H, *dvr = dv + t * H;
        for_columns<VEC, NT>(xr, H, [&](int j, bool vec) {
            if (vec) {
                float2 gf[4], xf[4], kf[4], a[4], b[4], cv[4];
                float w[8], pr[8];
                unpack4x2(*reinterpret_cast<const uint4 *>(gr + j), gf);
                unpack4x2(*reinterpret_cast<const uint4 *>(xr + j), xf);
                unpack4x2(*reinterpret_cast<const uint4 *>(kr + j), kf);
                if (SHIFT) wvec_at(wh, we, j, H, w_aligned, w);
                else wvec(wh, we, j, w);
                const bool acc4 = (reinterpret_cast<uintptr_t>(acc + j) & 15u) == 0;
                if (acc4) {
                    const float4 p0 = *reinterpret_cast<const float4 *>(acc + j);
                    const float4 p1 = *reinterpret_cast<const float4 *>(acc + j + 4);
                    pr[0] = p0.x; pr[1] = p0.y; pr[2] = p0.z; pr[3] = p0.w;
                    pr[4] = p1.x; pr[5] = p1.y; pr[6] = p1.z; pr[7] = p1.w;
                } else {
#pragma unroll
                    for (int e = 0; e < 8; ++e) pr[e] = acc[j + e];
                }
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float cw0 = c1 * w[2 * e], cw1 = c1 * w[2 * e + 1];
                    a[e] = make_float2(fmaf(-c2, xf[e].x, fmaf(cw0, kf[e].x, gf[e].x)),
                                       fmaf(-c2, xf[e].y, fmaf(cw1, kf[e].y, gf[e].y)));
                    b[e] = make_float2(fmaf(-c3, kf[e].x, cw0 * xf[e].x), fmaf(-c3, kf[e].y, cw1 * xf[e].y));
                    cv[e] = make_float2(c.gate * gf[e].x, c.gate * gf[e].y);
                    pr[2 * e] = fmaf(c1, xf[e].x * kf[e].x, pr[2 * e]);
                    pr[2 * e + 1] = fmaf(c1, xf[e].y * kf[e].y, pr[2 * e + 1]);
                }
                if (acc4) {
                    *reinterpret_cast<float4 *>(acc + j) = make_float4(pr[0], pr[1], pr[2], pr[3]);
                    *reinterpret_cast<float4 *>(acc + j + 4) = make_float4(pr[4], pr[5], pr[6], pr[7]);
                } else {
#pragma unroll
                    for (int e = 0; e < 8; ++e) acc[j + e] = pr[e];
                }
                __stcs(reinterpret_cast<uint4 *>(dxr + j), pack4x2(a));
                __stcs(reinterpret_cast<uint4 *>(dkr + j), pack4x2(b));
                __stcs(reinterpret_cast<uint4 *>(dvr + j), pack4x2(cv));
            } else {
                const float gv = bf(gr + j), xv = bf(xr + j), kv = bf(kr + j);
                const float cw = c1 * wcol(wh, we, j);
                dxr[j] = __float2bfloat16_rn(fmaf(-c2, xv, fmaf(cw, kv, gv)));
                dkr[j] = __float2bfloat16_rn(fmaf(-c3, kv, cw * xv));
                dvr[j] = __float2bfloat16_rn(c.gate * gv);
                acc[j] = fmaf(c1, xv * kv, acc[j]);
            }
        });
    }
    if (acc != prow) {
        __syncthreads();
        for (int j = threadIdx.x; j < H; j += NT) prow[j] = acc[j];
    }
}

}  // namespace engram
