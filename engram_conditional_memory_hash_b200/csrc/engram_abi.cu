// C ABI of the Engram hot path: argument checks, launch configuration and
// launches.  Declared in include/engram.h, which documents every call.
//
// All kernels live in this one translation unit (included below) so that the
// device error word has a single definition.
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "engram.h"

#include "common.cuh"
#include "gate_kernels.cuh"
#include "gather_bwd.cuh"
#include "hash_gather.cuh"

namespace {

thread_local char g_last_error[512] = "";

engram_status_t fail(engram_status_t st, const char *fmt, ...)
{
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_last_error, sizeof g_last_error, fmt, ap);
    va_end(ap);
    return st;
}

engram_status_t cuda_fail(cudaError_t e, const char *what)
{
    return fail(ENGRAM_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Per-device facts used to size the launches, read once per device.
struct DeviceInfo {
    int sms = 0;
    int smem_optin = 0;     // largest dynamic shared memory a CTA may opt into
    int smem_per_sm = 0;
};

constexpr int kMaxDevices = 64;
std::mutex g_dev_mutex;
DeviceInfo g_dev[kMaxDevices];
bool g_dev_ready[kMaxDevices];

engram_status_t device_info(DeviceInfo *out)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev < 0 || dev >= kMaxDevices) return fail(ENGRAM_ERR_UNSUPPORTED, "device ordinal %d", dev);
    std::lock_guard<std::mutex> lock(g_dev_mutex);
    if (!g_dev_ready[dev]) {
        DeviceInfo d;
        if ((e = cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess ||
            (e = cudaDeviceGetAttribute(&d.smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev)) !=
                cudaSuccess ||
            (e = cudaDeviceGetAttribute(&d.smem_per_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor,
                                        dev)) != cudaSuccess)
            return cuda_fail(e, "cudaDeviceGetAttribute");
        g_dev[dev] = d;
        g_dev_ready[dev] = true;
    }
    *out = g_dev[dev];
    return ENGRAM_OK;
}

// ------------------------------------------------------------ gate shape ----

constexpr int kGateMaxH = 8192;

// Launch shape of the gate kernels, chosen by timing launch shapes on B200 at
// H = 4096 and 7168: the forward runs 2 CTAs per SM of at most 256 threads
// (4 vectors per thread at H = 7168); the backward, whose registers hold four
// rows' worth of vectors plus the weight-gradient accumulators, runs one CTA
// per SM with 2 vectors per thread.  Overridable at compile time.
#ifndef ENGRAM_FWD_TARGET_THREADS
#define ENGRAM_FWD_TARGET_THREADS 256
#endif
#ifndef ENGRAM_FWD_MAX_CTAS
#define ENGRAM_FWD_MAX_CTAS 2
#endif
#ifndef ENGRAM_BWD_VEC
#define ENGRAM_BWD_VEC 2
#endif
#ifndef ENGRAM_BWD_MAX_CTAS
#define ENGRAM_BWD_MAX_CTAS 1
#endif
#ifndef ENGRAM_GATE_MAX_STAGES
#define ENGRAM_GATE_MAX_STAGES 8
#endif

struct GateLaunch {
    int maxv = 1;       // 16-byte column vectors per thread (1, 2 or 4)
    int threads = 32;
    int nstage = 2;
    size_t smem = 0;
    int ctas_per_sm = 1;
};

// Resident CTAs per SM of `kernel` with the given block and shared memory.
template <typename K>
engram_status_t occupancy(K kernel, int threads, size_t smem, int *n)
{
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(n, kernel, threads, smem);
    if (e != cudaSuccess) return cuda_fail(e, "cudaOccupancyMaxActiveBlocksPerMultiprocessor");
    return ENGRAM_OK;
}

// Shape of a gate kernel streaming `ntensors` rows of H bf16 per token with
// `maxv` vectors per thread: the most CTAs per SM (up to max_ctas) that still
// give each CTA at least two pipeline stages, with as many stages as the
// shared memory allows.
template <typename K1, typename K2, typename K4>
engram_status_t gate_plan(const DeviceInfo &d, int H, int ntensors, int maxv, int max_ctas, K1 k1,
                          K2 k2, K4 k4, GateLaunch *g)
{
    const int nvec = H / 8;
    g->maxv = maxv;
    g->threads = ((nvec + g->maxv - 1) / g->maxv + 31) / 32 * 32;
    const size_t stage = (size_t)ntensors * H * 2;
    for (int ctas = max_ctas; ctas >= 1; --ctas) {
        size_t budget = (size_t)d.smem_per_sm / ctas;
        budget = budget > 1024 ? budget - 1024 : 0;      // per-CTA reserved shared memory
        budget = std::min(budget, (size_t)d.smem_optin);
        if (budget <= engram::kGateRedBytes) continue;
        int ns = (int)((budget - engram::kGateRedBytes) / (stage + 8));
        ns = std::min(ns, ENGRAM_GATE_MAX_STAGES);
        if (ns < 2) continue;
        const size_t smem = engram::gate_smem_bytes(H, ntensors, ns);
        int n = 0;
        engram_status_t st = g->maxv == 1 ? occupancy(k1, g->threads, smem, &n)
                           : g->maxv == 2 ? occupancy(k2, g->threads, smem, &n)
                                          : occupancy(k4, g->threads, smem, &n);
        if (st != ENGRAM_OK) return st;
        if (n < 1) continue;
        g->nstage = ns;
        g->smem = smem;
        g->ctas_per_sm = std::min(n, ctas);
        return ENGRAM_OK;
    }
    return fail(ENGRAM_ERR_UNSUPPORTED, "H=%d: two pipeline stages of %zu B do not fit in shared memory",
                H, stage);
}

// Forward: the fewest vectors per thread that keep the CTA within the target.
engram_status_t gate_fwd_plan(const DeviceInfo &d, int H, GateLaunch *g)
{
    const int nvec = H / 8;
    int maxv = 4;
    for (int mv : {1, 2, 4}) {
        const int t = (nvec + mv - 1) / mv;
        if (t <= ENGRAM_FWD_TARGET_THREADS && t <= engram::gate_max_threads(mv)) {
            maxv = mv;
            break;
        }
    }
    return gate_plan(d, H, 3, maxv, ENGRAM_FWD_MAX_CTAS, engram::gate_fwd_kernel<1>,
                     engram::gate_fwd_kernel<2>, engram::gate_fwd_kernel<4>, g);
}

// Backward: ENGRAM_BWD_VEC vectors per thread (one for rows of at most 64
// vectors, four where two would need more than 512 threads).
engram_status_t gate_bwd_plan(const DeviceInfo &d, int H, GateLaunch *g)
{
    const int nvec = H / 8;
    int maxv = ENGRAM_BWD_VEC;
    if (nvec <= 64) maxv = 1;
    while ((nvec + maxv - 1) / maxv > engram::gate_max_threads(maxv) && maxv < 4) maxv *= 2;
    return gate_plan(d, H, 4, maxv, ENGRAM_BWD_MAX_CTAS, engram::gate_bwd_kernel<1>,
                     engram::gate_bwd_kernel<2>, engram::gate_bwd_kernel<4>, g);
}

engram_status_t check_gate_common(int64_t T, int32_t H, float eps, float scalar)
{
    if (T < 0) return fail(ENGRAM_ERR_INVALID_ARG, "T=%lld < 0", (long long)T);
    if (T > (int64_t(1) << 40)) return fail(ENGRAM_ERR_UNSUPPORTED, "T=%lld too large", (long long)T);
    if (H < 8 || H % 8 != 0 || H > kGateMaxH)
        return fail(ENGRAM_ERR_UNSUPPORTED, "H=%d: must be a multiple of 8 in [8, %d]", H, kGateMaxH);
    if (!std::isfinite(eps) || eps < 0.f) return fail(ENGRAM_ERR_INVALID_ARG, "eps must be finite and >= 0");
    if (!std::isfinite(scalar)) return fail(ENGRAM_ERR_INVALID_ARG, "scalar must be finite");
    return ENGRAM_OK;
}

// ------------------------------------------------------- gather backward ----

// Launch with programmatic stream serialisation: the kernel may be scheduled
// while the previous kernel of the stream drains; every kernel launched this
// way starts with pdl_wait_and_release(), so it reads nothing before its
// predecessor has completed.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), unsigned grid, unsigned block, cudaStream_t s,
                       Args... args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(block);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

constexpr int64_t kGbwdMaxEntries = int64_t(1) << 30;

// Offsets (bytes, 256-aligned) of the gather backward's scratch in the
// caller's workspace.  A region zeroed by every call first: the `seen` and
// `dupmap` bitmaps (one bit per table row) and the counters (list length,
// listed-chunk count).  Then the unique kernel's per-tile counts, two
// (key, position) buffers for the staged entries, the list and its radix
// passes (room for every entry), the digit histograms (for the larger of the
// staged and the list tilings) and totals, and the fp64 partial rows of
// chunk-crossing segments with the list of chunks where such segments end.
struct GbwdLayout {
    int64_t utiles = 0, stiles = 0, nchunks = 0, words = 0;
    size_t seen = 0, dupmap = 0, counters = 0, tile_cnt = 0;
    size_t keys_a = 0, vals_a = 0, keys_b = 0, vals_b = 0, hist = 0, totals = 0;
    size_t carry_a = 0, carry_b = 0, carry_list = 0;
    size_t total = 0;
    size_t zero_bytes() const { return tile_cnt - seen; }
};

GbwdLayout gbwd_layout(int64_t N, int D, int64_t R)
{
    GbwdLayout g;
    g.utiles = (N + engram::kUniqTile - 1) / engram::kUniqTile;
    g.stiles = (N + engram::kSortTile - 1) / engram::kSortTile;
    g.nchunks = (N + engram::kSegChunk - 1) / engram::kSegChunk;
    g.words = (R + 31) / 32;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t o = off;
        off = (off + bytes + 255) & ~size_t(255);
        return o;
    };
    g.seen = take((size_t)g.words * 4);
    g.dupmap = take((size_t)g.words * 4);
    g.counters = take(256);   // [0] list length M, [1] listed-chunk count
    g.tile_cnt = take((size_t)g.utiles * 4);
    g.keys_a = take((size_t)N * 4);
    g.vals_a = take((size_t)N * 4);
    g.keys_b = take((size_t)N * 4);
    g.vals_b = take((size_t)N * 4);
    g.hist = take((size_t)engram::kRadixBins * (size_t)std::max(g.stiles, g.utiles) * 4);
    g.totals = take((size_t)engram::kRadixBins * 4);
    g.carry_a = take((size_t)g.nchunks * (size_t)D * 8);
    g.carry_b = take((size_t)g.nchunks * (size_t)D * 8);
    g.carry_list = take((size_t)g.nchunks * 4);
    g.total = N > 0 ? off : 0;
    return g;
}

engram_status_t check_gbwd_sizes(int64_t T, int32_t L, int32_t J, int32_t D)
{
    if (T < 0) return fail(ENGRAM_ERR_INVALID_ARG, "T=%lld < 0", (long long)T);
    if (L < 1 || L > engram::kHashMaxL) return fail(ENGRAM_ERR_UNSUPPORTED, "L=%d not in [1, %d]", L, engram::kHashMaxL);
    if (J < 1 || J > engram::kHashMaxJ) return fail(ENGRAM_ERR_UNSUPPORTED, "J=%d not in [1, %d]", J, engram::kHashMaxJ);
    if (D < 8 || D > 256 || D % 8 != 0)
        return fail(ENGRAM_ERR_UNSUPPORTED, "D=%d: must be a multiple of 8 in [8, 256]", D);
    if (T > kGbwdMaxEntries / (L * J))
        return fail(ENGRAM_ERR_UNSUPPORTED, "T*L*J above 2^30 entries");
    return ENGRAM_OK;
}

}  // namespace

extern "C" {

int engram_abi_version(void) { return 1; }

const char *engram_status_string(engram_status_t status)
{
    switch (status) {
    case ENGRAM_OK: return "ok";
    case ENGRAM_ERR_INVALID_ARG: return "invalid argument";
    case ENGRAM_ERR_UNSUPPORTED: return "unsupported size";
    case ENGRAM_ERR_CUDA: return "CUDA runtime error";
    }
    return "unknown status";
}

const char *engram_last_error(void) { return g_last_error; }

// ------------------------------------------------------------ hash/gather ----

engram_status_t engram_hash_gather(const int64_t *tokens, int64_t B, int64_t S,
                                   const uint64_t *multipliers, const int32_t *ngram_n, int32_t L,
                                   int32_t n_max, const int64_t *table_sizes, int32_t J,
                                   const void *tables, int32_t D, int64_t pad_id, int64_t *idx_out,
                                   void *rows_out, engram_stream_t stream)
{
    using engram::HashParams;
    if (B < 0 || S < 0) return fail(ENGRAM_ERR_INVALID_ARG, "B=%lld, S=%lld", (long long)B, (long long)S);
    if (!multipliers || !ngram_n || !table_sizes)
        return fail(ENGRAM_ERR_INVALID_ARG, "multipliers, ngram_n and table_sizes are required");
    if (L < 1 || L > engram::kHashMaxL) return fail(ENGRAM_ERR_UNSUPPORTED, "L=%d not in [1, %d]", L, engram::kHashMaxL);
    if (J < 1 || J > engram::kHashMaxJ) return fail(ENGRAM_ERR_UNSUPPORTED, "J=%d not in [1, %d]", J, engram::kHashMaxJ);
    if (n_max < 1 || n_max > engram::kHashMaxN)
        return fail(ENGRAM_ERR_UNSUPPORTED, "n_max=%d not in [1, %d]", n_max, engram::kHashMaxN);
    if (B > 0 && S > 0 && B > (int64_t(1) << 40) / S) return fail(ENGRAM_ERR_UNSUPPORTED, "B*S too large");
    const int64_t T = B * S;
    if (T > 0 && !idx_out && !rows_out)
        return fail(ENGRAM_ERR_INVALID_ARG, "idx_out and rows_out are both NULL");
    if (rows_out && (D < 8 || D > 256 || D % 8 != 0))
        return fail(ENGRAM_ERR_UNSUPPORTED, "D=%d: must be a multiple of 8 in [8, 256]", D);

    HashParams p;
    std::memset(&p, 0, sizeof p);
    p.B = B;
    p.S = S;
    p.pad_id = pad_id;
    p.L = L;
    p.J = J;
    p.D = rows_out ? D : 8;
    int64_t total_rows = 0;
    for (int l = 0; l < L; ++l) {
        if (ngram_n[l] < 1 || ngram_n[l] > n_max)
            return fail(ENGRAM_ERR_INVALID_ARG, "ngram_n[%d]=%d not in [1, n_max=%d]", l, ngram_n[l], n_max);
        p.ngram_n[l] = ngram_n[l];
        for (int i = 0; i < n_max; ++i) p.mult[l][i] = multipliers[(int64_t)l * n_max + i];
        for (int j = 0; j < J; ++j) {
            const int q = l * J + j;
            const int64_t P = table_sizes[q];
            if (P < 1) return fail(ENGRAM_ERR_INVALID_ARG, "table_sizes[%d]=%lld < 1", q, (long long)P);
            p.P[q] = (uint64_t)P;
            p.inv[q] = ~uint64_t(0) / (uint64_t)P;
            p.row0[q] = total_rows;
            // the gather addresses rows of the concatenated tables with 64-bit
            // offsets of D * 2 bytes: keep the row count well inside that
            if (rows_out && P > (int64_t(1) << 48) - total_rows)
                return fail(ENGRAM_ERR_UNSUPPORTED, "total table rows exceed 2^48");
            total_rows += rows_out ? P : 0;
        }
    }
    if (T == 0) return ENGRAM_OK;
    if (!tokens) return fail(ENGRAM_ERR_INVALID_ARG, "tokens is NULL");
    if (!aligned(tokens, 8)) return fail(ENGRAM_ERR_INVALID_ARG, "tokens must be 8-byte aligned");
    if (idx_out && !aligned(idx_out, 8)) return fail(ENGRAM_ERR_INVALID_ARG, "idx_out must be 8-byte aligned");
    if (rows_out) {
        if (!tables) return fail(ENGRAM_ERR_INVALID_ARG, "tables is NULL");
        if (!aligned(tables, 16) || !aligned(rows_out, 16))
            return fail(ENGRAM_ERR_INVALID_ARG, "tables and rows_out must be 16-byte aligned");
    }

    DeviceInfo dev;
    engram_status_t st = device_info(&dev);
    if (st != ENGRAM_OK) return st;

    const int64_t ngroups = T * L;
    const int64_t groups_per_block = engram::kHashThreads / 8;
    int64_t blocks = (ngroups + groups_per_block - 1) / groups_per_block;
    blocks = std::min<int64_t>(blocks, (int64_t)dev.sms * 64);
    const int chunks = p.D / 8;
    const int cpl = (chunks + 7) / 8;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const uint4 *tab = static_cast<const uint4 *>(tables);
    uint4 *rows = static_cast<uint4 *>(rows_out);
    if (cpl <= 1)
        engram::hash_gather_kernel<1><<<(unsigned)blocks, engram::kHashThreads, 0, s>>>(tokens, tab, idx_out, rows, p);
    else if (cpl <= 2)
        engram::hash_gather_kernel<2><<<(unsigned)blocks, engram::kHashThreads, 0, s>>>(tokens, tab, idx_out, rows, p);
    else
        engram::hash_gather_kernel<4><<<(unsigned)blocks, engram::kHashThreads, 0, s>>>(tokens, tab, idx_out, rows, p);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "hash_gather launch");
    return ENGRAM_OK;
}

// ---------------------------------------------------------------- gate fwd ----

engram_status_t engram_gate_fwd(const void *x, const void *k, const void *v, const void *wh,
                                const void *we, int64_t T, int32_t H, float eps, float scalar,
                                void *out, float *gate, engram_stream_t stream)
{
    engram_status_t st = check_gate_common(T, H, eps, scalar);
    if (st != ENGRAM_OK) return st;
    if (T == 0) return ENGRAM_OK;
    if (!x || !k || !v || !wh || !we || !out)
        return fail(ENGRAM_ERR_INVALID_ARG, "x, k, v, wh, we and out are required");
    if (!aligned(x, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(wh, 16) || !aligned(we, 16) ||
        !aligned(out, 16))
        return fail(ENGRAM_ERR_INVALID_ARG, "bf16 tensors must be 16-byte aligned");
    if (gate && !aligned(gate, 4)) return fail(ENGRAM_ERR_INVALID_ARG, "gate must be 4-byte aligned");

    DeviceInfo dev;
    if ((st = device_info(&dev)) != ENGRAM_OK) return st;
    GateLaunch g;
    if ((st = gate_fwd_plan(dev, H, &g)) != ENGRAM_OK) return st;
    const int64_t grid = std::min<int64_t>(T, (int64_t)dev.sms * g.ctas_per_sm);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    auto args = [&](auto kern) -> engram_status_t {
        kern<<<(unsigned)grid, g.threads, g.smem, s>>>(
            static_cast<const uint4 *>(x), static_cast<const uint4 *>(k), static_cast<const uint4 *>(v),
            static_cast<const uint4 *>(wh), static_cast<const uint4 *>(we), T, H, eps, scalar,
            static_cast<uint4 *>(out), gate, g.nstage);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return cuda_fail(e, "gate_fwd launch");
        return ENGRAM_OK;
    };
    return g.maxv == 1 ? args(engram::gate_fwd_kernel<1>)
         : g.maxv == 2 ? args(engram::gate_fwd_kernel<2>)
                       : args(engram::gate_fwd_kernel<4>);
}

// ---------------------------------------------------------------- gate bwd ----

int64_t engram_gate_bwd_num_partials(int64_t T, int32_t H)
{
    if (H < 8 || H % 8 != 0 || H > kGateMaxH) {
        fail(ENGRAM_ERR_UNSUPPORTED, "H=%d: must be a multiple of 8 in [8, %d]", H, kGateMaxH);
        return -1;
    }
    DeviceInfo dev;
    if (device_info(&dev) != ENGRAM_OK) return -1;
    GateLaunch g;
    if (gate_bwd_plan(dev, H, &g) != ENGRAM_OK) return -1;
    const int64_t full = (int64_t)dev.sms * g.ctas_per_sm;
    return std::max<int64_t>(1, std::min<int64_t>(T, full));
}

engram_status_t engram_gate_bwd(const void *grad_out, const void *x, const void *k, const void *v,
                                const void *wh, const void *we, int64_t T, int32_t H, float eps,
                                float scalar, void *dx, void *dk, void *dv, float *w_partial, int64_t G,
                                engram_stream_t stream)
{
    engram_status_t st = check_gate_common(T, H, eps, scalar);
    if (st != ENGRAM_OK) return st;
    if (!wh || !we || !w_partial)
        return fail(ENGRAM_ERR_INVALID_ARG, "wh, we and w_partial are required");
    // with T == 0 the kernel only writes zero partial rows; the token tensors
    // may then be empty (NULL)
    if (T > 0 && (!grad_out || !x || !k || !v || !dx || !dk || !dv))
        return fail(ENGRAM_ERR_INVALID_ARG, "every tensor argument of engram_gate_bwd is required");
    if (G < 1 || G > 0x7fffffff) return fail(ENGRAM_ERR_INVALID_ARG, "G=%lld not in [1, 2^31-1]", (long long)G);
    if (!aligned(grad_out, 16) || !aligned(x, 16) || !aligned(k, 16) || !aligned(v, 16) ||
        !aligned(wh, 16) || !aligned(we, 16) || !aligned(dx, 16) || !aligned(dk, 16) ||
        !aligned(dv, 16) || !aligned(w_partial, 16))
        return fail(ENGRAM_ERR_INVALID_ARG, "tensors must be 16-byte aligned");

    DeviceInfo dev;
    if ((st = device_info(&dev)) != ENGRAM_OK) return st;
    GateLaunch g;
    if ((st = gate_bwd_plan(dev, H, &g)) != ENGRAM_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    auto args = [&](auto kern) -> engram_status_t {
        kern<<<(unsigned)G, g.threads, g.smem, s>>>(
            static_cast<const uint4 *>(grad_out), static_cast<const uint4 *>(x),
            static_cast<const uint4 *>(k), static_cast<const uint4 *>(v), static_cast<const uint4 *>(wh),
            static_cast<const uint4 *>(we), T, H, eps, scalar, static_cast<uint4 *>(dx),
            static_cast<uint4 *>(dk), static_cast<uint4 *>(dv), w_partial, g.nstage);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return cuda_fail(e, "gate_bwd launch");
        return ENGRAM_OK;
    };
    return g.maxv == 1 ? args(engram::gate_bwd_kernel<1>)
         : g.maxv == 2 ? args(engram::gate_bwd_kernel<2>)
                       : args(engram::gate_bwd_kernel<4>);
}

// ----------------------------------------------------------- grad_w_reduce ----

engram_status_t engram_grad_w_reduce(const float *w_partial, int64_t G, int32_t H, const void *wh,
                                     const void *we, float *dwh, float *dwe, engram_stream_t stream)
{
    if (G < 1 || G > 0x7fffffff) return fail(ENGRAM_ERR_INVALID_ARG, "G=%lld not in [1, 2^31-1]", (long long)G);
    if (H < 1) return fail(ENGRAM_ERR_INVALID_ARG, "H=%d < 1", H);
    if (!w_partial || !wh || !we || !dwh || !dwe)
        return fail(ENGRAM_ERR_INVALID_ARG, "every pointer argument of engram_grad_w_reduce is required");
    if (!aligned(w_partial, 4) || !aligned(dwh, 4) || !aligned(dwe, 4) || !aligned(wh, 2) || !aligned(we, 2))
        return fail(ENGRAM_ERR_INVALID_ARG, "misaligned pointer");
    const unsigned blocks = (unsigned)((H + 31) / 32);
    engram::grad_w_reduce_kernel<<<blocks, engram::kReduceThreads, 0,
                                   reinterpret_cast<cudaStream_t>(stream)>>>(
        w_partial, G, H, static_cast<const __nv_bfloat16 *>(wh), static_cast<const __nv_bfloat16 *>(we),
        dwh, dwe);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "grad_w_reduce launch");
    return ENGRAM_OK;
}

// -------------------------------------------------------- gather backward ----

int64_t engram_gather_bwd_workspace_size(int64_t T, int32_t L, int32_t J, int32_t D,
                                         int64_t total_rows)
{
    if (check_gbwd_sizes(T, L, J, D) != ENGRAM_OK) return -1;
    if (total_rows < 1 || total_rows > int64_t(0xfffffffe)) {
        fail(ENGRAM_ERR_UNSUPPORTED, "total_rows=%lld not in [1, 2^32 - 2]", (long long)total_rows);
        return -1;
    }
    return (int64_t)gbwd_layout(T * L * J, D, total_rows).total;   // 0 when T == 0
}

engram_status_t engram_gather_bwd(const int64_t *idx, int64_t T, int32_t L, int32_t J,
                                  const int64_t *table_sizes, const void *d_rows, int32_t D,
                                  float *d_tables, void *workspace, size_t workspace_bytes,
                                  engram_stream_t stream)
{
    using engram::GatherBwdParams;
    engram_status_t st = check_gbwd_sizes(T, L, J, D);
    if (st != ENGRAM_OK) return st;
    if (!table_sizes) return fail(ENGRAM_ERR_INVALID_ARG, "table_sizes is required");
    GatherBwdParams p;
    std::memset(&p, 0, sizeof p);
    p.LJ = L * J;
    p.D = D;
    int64_t R = 0;
    for (int q = 0; q < p.LJ; ++q) {
        const int64_t P = table_sizes[q];
        if (P < 1) return fail(ENGRAM_ERR_INVALID_ARG, "table_sizes[%d]=%lld < 1", q, (long long)P);
        if (P > int64_t(0xfffffffe) - R)
            return fail(ENGRAM_ERR_UNSUPPORTED, "total table rows must stay below 2^32 - 1");
        p.P[q] = (uint32_t)P;
        p.row0[q] = (uint32_t)R;
        R += P;
    }
    p.R = (uint32_t)R;
    const int64_t N = T * p.LJ;
    p.N = N;
    if (N == 0) return ENGRAM_OK;
    if (!idx || !d_rows || !d_tables || !workspace)
        return fail(ENGRAM_ERR_INVALID_ARG, "idx, d_rows, d_tables and workspace are required");
    if (!aligned(idx, 8)) return fail(ENGRAM_ERR_INVALID_ARG, "idx must be 8-byte aligned");
    if (!aligned(d_rows, 16) || !aligned(d_tables, 16) || !aligned(workspace, 16))
        return fail(ENGRAM_ERR_INVALID_ARG, "d_rows, d_tables and workspace must be 16-byte aligned");
    const GbwdLayout g = gbwd_layout(N, D, R);
    if (workspace_bytes < g.total)
        return fail(ENGRAM_ERR_INVALID_ARG, "workspace of %zu bytes, %zu needed", workspace_bytes, g.total);

    unsigned char *ws = static_cast<unsigned char *>(workspace);
    uint32_t *seen = reinterpret_cast<uint32_t *>(ws + g.seen);
    uint32_t *dupmap = reinterpret_cast<uint32_t *>(ws + g.dupmap);
    uint32_t *m_dev = reinterpret_cast<uint32_t *>(ws + g.counters);
    uint32_t *carry_count = m_dev + 1;
    uint32_t *tile_cnt = reinterpret_cast<uint32_t *>(ws + g.tile_cnt);
    uint32_t *keys[2] = {reinterpret_cast<uint32_t *>(ws + g.keys_a), reinterpret_cast<uint32_t *>(ws + g.keys_b)};
    uint32_t *vals[2] = {reinterpret_cast<uint32_t *>(ws + g.vals_a), reinterpret_cast<uint32_t *>(ws + g.vals_b)};
    uint32_t *hist = reinterpret_cast<uint32_t *>(ws + g.hist);
    uint32_t *totals = reinterpret_cast<uint32_t *>(ws + g.totals);
    double *carry_a = reinterpret_cast<double *>(ws + g.carry_a);
    double *carry_b = reinterpret_cast<double *>(ws + g.carry_b);
    uint32_t *carry_list = reinterpret_cast<uint32_t *>(ws + g.carry_list);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const uint4 *rows = static_cast<const uint4 *>(d_rows);
    float4 *tab4 = reinterpret_cast<float4 *>(d_tables);
    const uint32_t *m_c = m_dev;
    const int nv = D / 8;   // 16-byte vectors per row: lanes per group

    cudaError_t e = cudaMemsetAsync(ws + g.seen, 0, g.zero_bytes(), s);
    // 1. mark rows read more than once
    if (e == cudaSuccess) {
        const unsigned mblocks = (unsigned)std::min<int64_t>(
            (N + 4 * engram::kMarkThreads - 1) / (4 * engram::kMarkThreads), 4096);
        e = launch_pdl(engram::gbwd_mark_kernel, mblocks, (unsigned)engram::kMarkThreads, s, idx, p, seen,
                       dupmap);
    }
    // 2. rows read once: update in place; stage the rest per tile (into the
    //    second buffer pair), with the first radix pass's tile histograms
    if (e == cudaSuccess) {
        const unsigned ub = (unsigned)g.utiles, ut = (unsigned)engram::kUniqThreads;
        const uint32_t *dm = dupmap;
        if (nv <= 4)
            e = launch_pdl(engram::gbwd_unique_kernel<4, 4>, ub, ut, s, idx, rows, p, dm, tab4, keys[1], vals[1],
                           tile_cnt, hist, m_dev);
        else if (nv <= 8)
            e = launch_pdl(engram::gbwd_unique_kernel<8, 4>, ub, ut, s, idx, rows, p, dm, tab4, keys[1], vals[1],
                           tile_cnt, hist, m_dev);
        else if (nv <= 16)
            e = launch_pdl(engram::gbwd_unique_kernel<16, 4>, ub, ut, s, idx, rows, p, dm, tab4, keys[1],
                           vals[1], tile_cnt, hist, m_dev);
        else
            e = launch_pdl(engram::gbwd_unique_kernel<32, 4>, ub, ut, s, idx, rows, p, dm, tab4, keys[1],
                           vals[1], tile_cnt, hist, m_dev);
    }
    // 3. stable radix sort by row of the staged entries into a contiguous
    //    list; keys lie in [0, R): sort on the bit length of R - 1
    int nbits = 0;
    while (nbits < 32 && (uint64_t(R - 1) >> nbits) != 0) ++nbits;
    const int npasses = std::max(1, (nbits + 7) / 8);
    const unsigned stiles = (unsigned)g.stiles, T_ = engram::kSortThreads;
    const uint32_t *no_cnt = nullptr;
    int cur = 1;   // the staged entries are in the second buffer pair
    for (int pass = 0; pass < npasses && e == cudaSuccess; ++pass) {
        const int shift = 8 * pass;
        if (pass > 0)
            e = launch_pdl(engram::gbwd_hist_kernel, stiles, T_, s, static_cast<const uint32_t *>(keys[cur]),
                           m_c, shift, hist);
        if (e == cudaSuccess)
            e = launch_pdl(engram::gbwd_digit_scan_kernel, (unsigned)engram::kRadixBins,
                           (unsigned)engram::kScanThreads, s, hist, m_c, pass == 0 ? g.utiles : int64_t(0),
                           totals);
        if (e == cudaSuccess)
            e = launch_pdl(engram::gbwd_scatter_kernel, pass == 0 ? (unsigned)g.utiles : stiles, T_, s,
                           static_cast<const uint32_t *>(keys[cur]), static_cast<const uint32_t *>(vals[cur]),
                           m_c, pass == 0 ? static_cast<const uint32_t *>(tile_cnt) : no_cnt, shift,
                           static_cast<const uint32_t *>(hist), static_cast<const uint32_t *>(totals),
                           keys[1 - cur], vals[1 - cur]);
        cur = 1 - cur;
    }
    // 4. segments of the sorted list, then the segments that cross chunks
    const int64_t seg_blocks = (g.nchunks + engram::kSegThreads / 32 - 1) / (engram::kSegThreads / 32);
    const unsigned blocks = (unsigned)std::min<int64_t>(seg_blocks, int64_t(1) << 30);
    const unsigned S_ = engram::kSegThreads;
    const uint32_t *kc = keys[cur], *vc = vals[cur];
    if (e == cudaSuccess) {
        if (nv <= 4)
            e = launch_pdl(engram::gbwd_segment_kernel<4, 2>, blocks, S_, s, kc, vc, rows, p, tab4, carry_a,
                           carry_b, carry_list, carry_count, m_c);
        else if (nv <= 8)
            e = launch_pdl(engram::gbwd_segment_kernel<8, 2>, blocks, S_, s, kc, vc, rows, p, tab4, carry_a,
                           carry_b, carry_list, carry_count, m_c);
        else if (nv <= 16)
            e = launch_pdl(engram::gbwd_segment_kernel<16, 2>, blocks, S_, s, kc, vc, rows, p, tab4, carry_a,
                           carry_b, carry_list, carry_count, m_c);
        else
            e = launch_pdl(engram::gbwd_segment_kernel<32, 2>, blocks, S_, s, kc, vc, rows, p, tab4, carry_a,
                           carry_b, carry_list, carry_count, m_c);
    }
    // one warp per listed chunk (a warp loops when more than 4096 are listed)
    const int64_t carry_warps = std::min<int64_t>(g.nchunks, 4096);
    const unsigned carry_blocks = (unsigned)((carry_warps + engram::kCarryThreads / 32 - 1) /
                                             (engram::kCarryThreads / 32));
    const unsigned CT = engram::kCarryThreads;
    const double *ca = carry_a, *cb = carry_b;
    const uint32_t *cl = carry_list, *cn = carry_count;
    if (e == cudaSuccess) {
        if (D <= 32)
            e = launch_pdl(engram::gbwd_carry_kernel<1>, carry_blocks, CT, s, kc, p, d_tables, ca, cb, cl, cn);
        else if (D <= 64)
            e = launch_pdl(engram::gbwd_carry_kernel<2>, carry_blocks, CT, s, kc, p, d_tables, ca, cb, cl, cn);
        else if (D <= 128)
            e = launch_pdl(engram::gbwd_carry_kernel<4>, carry_blocks, CT, s, kc, p, d_tables, ca, cb, cl, cn);
        else
            e = launch_pdl(engram::gbwd_carry_kernel<8>, carry_blocks, CT, s, kc, p, d_tables, ca, cb, cl, cn);
    }
    if (e != cudaSuccess) return cuda_fail(e, "gather_bwd launch");
    return ENGRAM_OK;
}

// ------------------------------------------------------------ diagnostics ----

engram_status_t engram_read_device_error(uint32_t *code_out, int32_t clear)
{
    if (!code_out) return fail(ENGRAM_ERR_INVALID_ARG, "code_out is NULL");
    cudaError_t e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceSynchronize");
    unsigned int v = 0;
    e = cudaMemcpyFromSymbol(&v, engram::g_device_error, sizeof v);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpyFromSymbol");
    if (clear) {
        const unsigned int zero = 0;
        e = cudaMemcpyToSymbol(engram::g_device_error, &zero, sizeof zero);
        if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpyToSymbol");
    }
    *code_out = v;
    return ENGRAM_OK;
}

}  // extern "C"

// ------------------------------------------------------ allocation-free bwd ----
//
// engram_gate_bwd_noalloc: engram_gate_bwd followed by engram_grad_w_reduce
// for callers that cannot allocate device memory (for example code running
// under a memory-pool policy that forbids cudaMalloc, or a host runtime whose
// only device buffers are the ones it was handed).  The
// weight-gradient partial rows, the only scratch of the backward, live in the
// fixed array below instead of a caller-provided buffer.

// Scratch: partial rows of the weight-gradient reduction, at most
// kNoAllocPartialFloats fp32 values (8 MiB).  Every GPU that loads this
// library holds the array until the process exits.
static constexpr size_t kNoAllocPartialFloats = size_t(1) << 21;
static __device__ __align__(256) float g_noalloc_partials[kNoAllocPartialFloats];

namespace {

std::mutex g_noalloc_mutex;
float *g_noalloc_ptr[kMaxDevices];

// Device address of g_noalloc_partials on the current device.  The name of
// the array in host code is only a host-side stand-in, so the address is
// looked up once per device (with that device current) and cached.
engram_status_t noalloc_scratch(float **out)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev < 0 || dev >= kMaxDevices) return fail(ENGRAM_ERR_UNSUPPORTED, "device ordinal %d", dev);
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    if (g_noalloc_ptr[dev] == nullptr) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_partials);
        if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress");
        g_noalloc_ptr[dev] = static_cast<float *>(p);
    }
    *out = g_noalloc_ptr[dev];
    return ENGRAM_OK;
}

}  // namespace

extern "C" engram_status_t engram_gate_bwd_noalloc(const void *grad_out, const void *x, const void *k,
                                                   const void *v, const void *wh, const void *we,
                                                   int64_t T, int32_t H, float eps, float scalar,
                                                   void *dx, void *dk, void *dv, float *dwh,
                                                   float *dwe, engram_stream_t stream)
{
    engram_status_t st = check_gate_common(T, H, eps, scalar);
    if (st != ENGRAM_OK) return st;
    if (!dwh || !dwe) return fail(ENGRAM_ERR_INVALID_ARG, "dwh and dwe are required");
    if (!aligned(dwh, 4) || !aligned(dwe, 4))
        return fail(ENGRAM_ERR_INVALID_ARG, "dwh and dwe must be 4-byte aligned");
    const int64_t G = engram_gate_bwd_num_partials(T, H);
    if (G < 1) return ENGRAM_ERR_CUDA;  // message set by engram_gate_bwd_num_partials
    if ((size_t)G * (size_t)H > kNoAllocPartialFloats)
        return fail(ENGRAM_ERR_UNSUPPORTED,
                    "engram_gate_bwd_noalloc: %lld partial rows x H=%d need %lld floats of scratch, "
                    "more than its static maximum of %zu",
                    (long long)G, H, (long long)(G * H), kNoAllocPartialFloats);
    float *scratch = nullptr;
    if ((st = noalloc_scratch(&scratch)) != ENGRAM_OK) return st;
    // Every partial row the reduction reads is written by the backward first
    // (rows of CTAs without tokens as zeros), so nothing has to be cleared.
    st = engram_gate_bwd(grad_out, x, k, v, wh, we, T, H, eps, scalar, dx, dk, dv, scratch, G, stream);
    if (st != ENGRAM_OK) return st;
    return engram_grad_w_reduce(scratch, G, H, wh, we, dwh, dwe, stream);
}
