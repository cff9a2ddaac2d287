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
#include <initializer_list>
#include <map>
#include <mutex>
#include <utility>

#include "engram.h"

#include "common.cuh"
#include "gate_generic.cuh"
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
    int ordinal = 0;
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
        d.ordinal = dev;
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
// H = 4096 and 7168: the forward runs CTAs of at most 256 threads (4 vectors
// per thread at H = 7168), as many per SM as registers allow up to 4, with the
// shared memory split between them (2 CTAs at both sizes; at H = 4096 that
// leaves 2 pipeline stages each, 86.5 us per forward of 16384 tokens against
// 96.9 with 4 stages when the cap was 2 CTAs); the backward, whose registers
// hold four rows' worth of vectors plus the weight-gradient accumulators, runs
// one CTA per SM with 2 vectors per thread.  Overridable at compile time.
#ifndef ENGRAM_FWD_TARGET_THREADS
#define ENGRAM_FWD_TARGET_THREADS 256
#endif
#ifndef ENGRAM_FWD_MAX_CTAS
#define ENGRAM_FWD_MAX_CTAS 4
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
// The kernel's shared-memory opt-in is raised to `smem` and never lowered, so
// that a launch sized by an earlier (cached) plan stays valid.
template <typename K>
engram_status_t occupancy(K kernel, int threads, size_t smem, int *n)
{
    cudaFuncAttributes fa;
    cudaError_t e = cudaFuncGetAttributes(&fa, kernel);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncGetAttributes");
    if ((size_t)fa.maxDynamicSharedSizeBytes < smem)
        e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
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

// Thread bound of the two-vector backward variant with the larger register
// budget (used whenever the row needs no more threads).
constexpr int kBwdNarrowThreads = 448;

// Backward: ENGRAM_BWD_VEC vectors per thread (one for rows of at most 64
// vectors, four where two would need more than 512 threads).
engram_status_t gate_bwd_plan(const DeviceInfo &d, int H, GateLaunch *g)
{
    const int nvec = H / 8;
    int maxv = ENGRAM_BWD_VEC;
    if (nvec <= 64) maxv = 1;
    while ((nvec + maxv - 1) / maxv > engram::gate_max_threads(maxv) && maxv < 4) maxv *= 2;
    if (maxv == 2 && (nvec + 1) / 2 <= kBwdNarrowThreads)
        return gate_plan(d, H, 4, maxv, ENGRAM_BWD_MAX_CTAS, engram::gate_bwd_kernel<1>,
                         engram::gate_bwd_kernel<2, kBwdNarrowThreads>, engram::gate_bwd_kernel<4>, g);
    return gate_plan(d, H, 4, maxv, ENGRAM_BWD_MAX_CTAS, engram::gate_bwd_kernel<1>,
                     engram::gate_bwd_kernel<2>, engram::gate_bwd_kernel<4>, g);
}

// The plans, computed once per device, hidden size and direction: planning
// sets the kernels' shared-memory attributes and queries the occupancy API,
// host calls that cost time on every launch otherwise (and setting an
// attribute of a kernel that is still running can make the host wait for it,
// leaving the GPU idle between calls).  The fused backward's attribute is set
// here too, once.
std::mutex g_plan_mutex;
std::map<std::pair<int, int>, GateLaunch> g_plans;   // (ordinal * 2 + direction, H)

engram_status_t set_fused_bwd_attribute(const GateLaunch &g);

engram_status_t cached_gate_plan(const DeviceInfo &d, int H, bool backward, GateLaunch *g)
{
    const std::pair<int, int> key(d.ordinal * 2 + (backward ? 1 : 0), H);
    std::lock_guard<std::mutex> lock(g_plan_mutex);
    auto it = g_plans.find(key);
    if (it != g_plans.end()) {
        *g = it->second;
        return ENGRAM_OK;
    }
    engram_status_t st = backward ? gate_bwd_plan(d, H, g) : gate_fwd_plan(d, H, g);
    if (st == ENGRAM_OK && backward) st = set_fused_bwd_attribute(*g);
    if (st == ENGRAM_OK) g_plans.emplace(key, *g);
    return st;
}

// Resident CTAs per SM of hash_gather_kernel<1|2|4> (variant 0|1|2) on device
// d, looked up once per device and variant.
std::mutex g_hg_mutex;
int g_hg_resident[kMaxDevices][3];

engram_status_t hash_gather_residency(const DeviceInfo &d, int variant, int *n)
{
    std::lock_guard<std::mutex> lock(g_hg_mutex);
    int &r = g_hg_resident[d.ordinal][variant];
    if (r == 0) {
        engram_status_t st = variant == 0 ? occupancy(engram::hash_gather_kernel<1>, engram::kHashThreads, 0, &r)
                             : variant == 1 ? occupancy(engram::hash_gather_kernel<2>, engram::kHashThreads, 0, &r)
                                            : occupancy(engram::hash_gather_kernel<4>, engram::kHashThreads, 0, &r);
        if (st != ENGRAM_OK) {
            r = 0;
            return st;
        }
    }
    *n = r;
    return ENGRAM_OK;
}

engram_status_t check_gate_common(int64_t T, int32_t H, float eps, float scalar)
{
    if (T < 0) return fail(ENGRAM_ERR_INVALID_ARG, "T=%lld < 0", (long long)T);
    if (T > (int64_t(1) << 40)) return fail(ENGRAM_ERR_UNSUPPORTED, "T=%lld too large", (long long)T);
    if (H < 1 || H > engram::kGenMaxH)
        return fail(ENGRAM_ERR_UNSUPPORTED, "H=%d not in [1, %d]", H, engram::kGenMaxH);
    if (!std::isfinite(eps) || eps < 0.f) return fail(ENGRAM_ERR_INVALID_ARG, "eps must be finite and >= 0");
    if (!std::isfinite(scalar)) return fail(ENGRAM_ERR_INVALID_ARG, "scalar must be finite");
    return ENGRAM_OK;
}

// The tuned gate kernels stream whole rows with 16-byte bulk copies: H a
// multiple of 8 up to kGateMaxH and every bf16 tensor on a 16-byte boundary.
// Any other H (up to kGenMaxH) or 2-byte alignment goes to gate_generic.cuh.
bool gate_tuned(int H, std::initializer_list<const void *> ptrs)
{
    if (H % 8 != 0 || H > kGateMaxH) return false;
    for (const void *p : ptrs)
        if (p != nullptr && !aligned(p, 16)) return false;
    return true;
}

// The generic kernels read rows with 16-byte vectors when every token tensor
// starts at the same offset from a 16-byte boundary.
bool same_phase(std::initializer_list<const void *> ptrs)
{
    int phase = -1;
    for (const void *p : ptrs) {
        if (p == nullptr) continue;
        const int ph = (int)(reinterpret_cast<uintptr_t>(p) & 15u);
        if (phase < 0) phase = ph;
        else if (ph != phase) return false;
    }
    return true;
}

// The generic kernel variant for rows of H values: VEC (token tensors share
// their offset from a 16-byte boundary), SHIFT (see shifted_rows) and the
// block size gen_threads(H).
using GenFwdKernel = void (*)(const __nv_bfloat16 *, const __nv_bfloat16 *, const __nv_bfloat16 *,
                              const __nv_bfloat16 *, const __nv_bfloat16 *, int64_t, int, float, float,
                              __nv_bfloat16 *, float *);
using GenBwdKernel = void (*)(const __nv_bfloat16 *, const __nv_bfloat16 *, const __nv_bfloat16 *,
                              const __nv_bfloat16 *, const __nv_bfloat16 *, const __nv_bfloat16 *, int64_t, int,
                              float, float, __nv_bfloat16 *, __nv_bfloat16 *, __nv_bfloat16 *, float *);

template <int NT>
GenFwdKernel gen_fwd_variant(bool vec, bool shift)
{
    using namespace engram;
    return !vec ? gate_generic_fwd_kernel<false, false, NT>
         : shift ? gate_generic_fwd_kernel<true, true, NT> : gate_generic_fwd_kernel<true, false, NT>;
}

template <int NT>
GenBwdKernel gen_bwd_variant(bool vec, bool shift)
{
    using namespace engram;
    return !vec ? gate_generic_bwd_kernel<false, false, NT>
         : shift ? gate_generic_bwd_kernel<true, true, NT> : gate_generic_bwd_kernel<true, false, NT>;
}

GenFwdKernel gen_fwd_kernel(int H, bool vec, bool shift)
{
    const int nt = engram::gen_threads(H);
    return nt == 64 ? gen_fwd_variant<64>(vec, shift)
         : nt == 128 ? gen_fwd_variant<128>(vec, shift) : gen_fwd_variant<256>(vec, shift);
}

GenBwdKernel gen_bwd_kernel(int H, bool vec, bool shift)
{
    const int nt = engram::gen_threads(H);
    return nt == 64 ? gen_bwd_variant<64>(vec, shift)
         : nt == 128 ? gen_bwd_variant<128>(vec, shift) : gen_bwd_variant<256>(vec, shift);
}

// Whether some token row of a tensor starting at `x` with rows of H values has
// its 16-byte vectors off the 16-byte boundaries of wh and we (odd rows, or a
// tensor past a boundary): the generic kernels then build the fused weight
// from aligned chunks (SHIFT).
bool shifted_rows(int H, const void *x) { return (H % 8) != 0 || !aligned(x, 16); }

// CTAs of a generic gate kernel: as many as the SMs hold at once (one wave),
// never more than tokens.
template <typename K>
engram_status_t generic_grid(const DeviceInfo &d, int64_t T, int H, K kernel, size_t smem, int64_t *grid)
{
    int n = 0;
    engram_status_t st = occupancy(kernel, engram::gen_threads(H), smem, &n);
    if (st != ENGRAM_OK) return st;
    *grid = std::max<int64_t>(1, std::min<int64_t>(T, (int64_t)d.sms * std::max(n, 1)));
    return ENGRAM_OK;
}

// Dynamic shared memory of the generic backward: its partial row, when it fits.
// Dynamic shared memory of the generic backward: its partial row, when it
// fits, with 8 floats of room for the padding of shifted rows, exactly H
// floats otherwise.  (At H = 16384, three CTAs per SM, 32 more bytes per CTA
// made the backward of 16384 tokens take 972 us instead of 806 us: same
// instructions, same occupancy, a lower L1 hit rate; presumably the CTAs'
// shared memory then no longer fits the smaller carveout, leaving less L1.)
size_t generic_bwd_smem(int H, bool shift) { return H <= engram::kGenSmemPartial ? (size_t)(H + (shift ? 8 : 0)) * 4 : 0; }

// Partial rows (CTAs) of the generic backward: one wave of the kernel variant
// with the fewer resident CTAs per SM, rounded down to a multiple of
// 8 / gcd(H, 8) so that G * H is a multiple of 8: then every token row of a
// CTA starts at the same offset from a 16-byte boundary (rows c, c + G, ...
// are G * H values apart) and the CTA's partial row can be laid out for
// 16-byte access (see gate_generic_bwd_kernel).
engram_status_t generic_bwd_grid(const DeviceInfo &d, int64_t T, int H, int64_t *grid)
{
    int64_t a = 0, b = 0;
    const size_t smem = generic_bwd_smem(H, true);
    int64_t c = 0;
    engram_status_t st = generic_grid(d, T, H, gen_bwd_kernel(H, true, true), smem, &a);
    if (st == ENGRAM_OK) st = generic_grid(d, T, H, gen_bwd_kernel(H, true, false), smem, &b);
    if (st == ENGRAM_OK) st = generic_grid(d, T, H, gen_bwd_kernel(H, false, false), smem, &c);
    int64_t g = std::min(std::min(a, b), c);
    const int64_t m = 8 / ((H & 7) == 0 ? 8 : (H & 3) == 0 ? 4 : (H & 1) == 0 ? 2 : 1);
    if (g >= m) g -= g % m;
    *grid = g;
    return st;
}

// -------------------------------------------------------------- launches ----

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

// Launch of the tuned backward kernel; with tickets != NULL the kernel also
// reduces the partial rows into dwh, dwe in its tail (engram_gate_bwd_fused).
engram_status_t launch_gate_bwd_tuned(const DeviceInfo &dev, const void *grad_out, const void *x,
                                      const void *k, const void *v, const void *wh, const void *we,
                                      int64_t T, int32_t H, float eps, float scalar, void *dx, void *dk,
                                      void *dv, float *w_partial, int64_t G, unsigned int *tickets,
                                      float *dwh, float *dwe, cudaStream_t s)
{
    GateLaunch g;
    engram_status_t st = cached_gate_plan(dev, H, true, &g);
    if (st != ENGRAM_OK) return st;
    const engram::ReduceGroups grp = engram::reduce_groups(G);
    // CTAs of the fused tail that may wait for the others: half of those the
    // GPU holds at once
    const int kmax = std::max(1, dev.sms * g.ctas_per_sm / 2);
    auto args = [&](auto kern) -> engram_status_t {
        kern<<<(unsigned)G, g.threads, g.smem, s>>>(
            static_cast<const uint4 *>(grad_out), static_cast<const uint4 *>(x),
            static_cast<const uint4 *>(k), static_cast<const uint4 *>(v), static_cast<const uint4 *>(wh),
            static_cast<const uint4 *>(we), T, H, eps, scalar, static_cast<uint4 *>(dx),
            static_cast<uint4 *>(dk), static_cast<uint4 *>(dv), w_partial, g.nstage, tickets, grp, kmax, dwh,
            dwe);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return cuda_fail(e, "gate_bwd launch");
        return ENGRAM_OK;
    };
    using engram::gate_bwd_kernel;
    constexpr int M1 = engram::gate_max_threads(1), M2 = engram::gate_max_threads(2),
                  M4 = engram::gate_max_threads(4);
    if (tickets != nullptr) {
        if (g.maxv == 2 && g.threads <= kBwdNarrowThreads) return args(gate_bwd_kernel<2, kBwdNarrowThreads, true>);
        return g.maxv == 1 ? args(gate_bwd_kernel<1, M1, true>)
             : g.maxv == 2 ? args(gate_bwd_kernel<2, M2, true>)
                           : args(gate_bwd_kernel<4, M4, true>);
    }
    if (g.maxv == 2 && g.threads <= kBwdNarrowThreads) return args(gate_bwd_kernel<2, kBwdNarrowThreads>);
    return g.maxv == 1 ? args(gate_bwd_kernel<1>)
         : g.maxv == 2 ? args(gate_bwd_kernel<2>)
                       : args(gate_bwd_kernel<4>);
}

// The shared-memory opt-in of the fused backward variant that a plan launches
// (the plan itself sized the launch on the plain kernel).
engram_status_t set_fused_bwd_attribute(const GateLaunch &g)
{
    using engram::gate_bwd_kernel;
    constexpr int M1 = engram::gate_max_threads(1), M2 = engram::gate_max_threads(2),
                  M4 = engram::gate_max_threads(4);
    auto set = [&](auto kern) -> engram_status_t {
        int n = 0;
        return occupancy(kern, g.threads, g.smem, &n);   // raises the opt-in to g.smem
    };
    if (g.maxv == 2 && g.threads <= kBwdNarrowThreads) return set(gate_bwd_kernel<2, kBwdNarrowThreads, true>);
    return g.maxv == 1 ? set(gate_bwd_kernel<1, M1, true>)
         : g.maxv == 2 ? set(gate_bwd_kernel<2, M2, true>)
                       : set(gate_bwd_kernel<4, M4, true>);
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
    p.inv_L = ~uint64_t(0) / (uint64_t)L;
    p.inv_S = ~uint64_t(0) / (uint64_t)S;
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
    const int chunks = p.D / 8;
    const int cpl = (chunks + 7) / 8;
    const int variant = cpl <= 1 ? 0 : cpl <= 2 ? 1 : 2;
    int resident = 0;
    if ((st = hash_gather_residency(dev, variant, &resident)) != ENGRAM_OK) return st;
    // The full grid (one CTA per 32 (token, layer) groups) unless it spans at
    // most four waves of resident CTAs and ends on a wave less than 3/4 full:
    // then one wave loops over the groups instead (T = 32768 at the hash-gather
    // tables: 24.8 us against 26.3 us with the full grid's 3.46 waves; the
    // full path's 6.9 waves stay: one looping wave took 51.5 against 48.3 us).
    const int64_t full = (ngroups + groups_per_block - 1) / groups_per_block;
    const int64_t wave = (int64_t)dev.sms * resident;
    int64_t blocks = full;
    if (wave > 0 && full > wave && full <= 4 * wave) {
        const int64_t last = full - (full - 1) / wave * wave;   // CTAs in the last wave
        if (4 * last < 3 * wave) blocks = wave;
    }
    blocks = std::min<int64_t>(blocks, (int64_t)dev.sms * 64);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const uint4 *tab = static_cast<const uint4 *>(tables);
    uint4 *rows = static_cast<uint4 *>(rows_out);
    if (variant == 0)
        engram::hash_gather_kernel<1><<<(unsigned)blocks, engram::kHashThreads, 0, s>>>(tokens, tab, idx_out, rows, p);
    else if (variant == 1)
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
    if (!aligned(x, 2) || !aligned(k, 2) || !aligned(v, 2) || !aligned(wh, 2) || !aligned(we, 2) ||
        !aligned(out, 2))
        return fail(ENGRAM_ERR_INVALID_ARG, "bf16 tensors must be 2-byte aligned");
    if (gate && !aligned(gate, 4)) return fail(ENGRAM_ERR_INVALID_ARG, "gate must be 4-byte aligned");

    DeviceInfo dev;
    if ((st = device_info(&dev)) != ENGRAM_OK) return st;
    if (!gate_tuned(H, {x, k, v, wh, we, out})) {
        const GenFwdKernel kern = gen_fwd_kernel(H, same_phase({x, k, v, out}), shifted_rows(H, x));
        int64_t grid = 0;
        if ((st = generic_grid(dev, T, H, kern, 0, &grid)) != ENGRAM_OK) return st;
        kern<<<(unsigned)grid, engram::gen_threads(H), 0, reinterpret_cast<cudaStream_t>(stream)>>>(
            static_cast<const __nv_bfloat16 *>(x), static_cast<const __nv_bfloat16 *>(k),
            static_cast<const __nv_bfloat16 *>(v), static_cast<const __nv_bfloat16 *>(wh),
            static_cast<const __nv_bfloat16 *>(we), T, H, eps, scalar, static_cast<__nv_bfloat16 *>(out),
            gate);
        const cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return cuda_fail(e, "gate_fwd launch");
        return ENGRAM_OK;
    }
    GateLaunch g;
    if ((st = cached_gate_plan(dev, H, false, &g)) != ENGRAM_OK) return st;
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
    if (H < 1 || H > engram::kGenMaxH) {
        fail(ENGRAM_ERR_UNSUPPORTED, "H=%d not in [1, %d]", H, engram::kGenMaxH);
        return -1;
    }
    DeviceInfo dev;
    if (device_info(&dev) != ENGRAM_OK) return -1;
    if (!gate_tuned(H, {})) {
        int64_t grid = 0;
        return generic_bwd_grid(dev, T, H, &grid) == ENGRAM_OK ? grid : -1;
    }
    GateLaunch g;
    if (cached_gate_plan(dev, H, true, &g) != ENGRAM_OK) return -1;
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
    if (!aligned(grad_out, 2) || !aligned(x, 2) || !aligned(k, 2) || !aligned(v, 2) || !aligned(wh, 2) ||
        !aligned(we, 2) || !aligned(dx, 2) || !aligned(dk, 2) || !aligned(dv, 2))
        return fail(ENGRAM_ERR_INVALID_ARG, "bf16 tensors must be 2-byte aligned");
    if (!aligned(w_partial, 4)) return fail(ENGRAM_ERR_INVALID_ARG, "w_partial must be 4-byte aligned");

    DeviceInfo dev;
    if ((st = device_info(&dev)) != ENGRAM_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (!gate_tuned(H, {grad_out, x, k, v, wh, we, dx, dk, dv, w_partial})) {
        const GenBwdKernel kern =
            gen_bwd_kernel(H, same_phase({grad_out, x, k, v, dx, dk, dv}), shifted_rows(H, x));
        const size_t smem = generic_bwd_smem(H, shifted_rows(H, x));
        int unused = 0;
        if ((st = occupancy(kern, engram::gen_threads(H), smem, &unused)) != ENGRAM_OK) return st;
        kern<<<(unsigned)G, engram::gen_threads(H), smem, s>>>(
            static_cast<const __nv_bfloat16 *>(grad_out), static_cast<const __nv_bfloat16 *>(x),
            static_cast<const __nv_bfloat16 *>(k), static_cast<const __nv_bfloat16 *>(v),
            static_cast<const __nv_bfloat16 *>(wh), static_cast<const __nv_bfloat16 *>(we), T, H, eps, scalar,
            static_cast<__nv_bfloat16 *>(dx), static_cast<__nv_bfloat16 *>(dk),
            static_cast<__nv_bfloat16 *>(dv), w_partial);
        const cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return cuda_fail(e, "gate_bwd launch");
        return ENGRAM_OK;
    }
    return launch_gate_bwd_tuned(dev, grad_out, x, k, v, wh, we, T, H, eps, scalar, dx, dk, dv, w_partial,
                                 G, nullptr, nullptr, nullptr, s);
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
    // programmatic launch: scheduled while the backward kernel drains
    const cudaError_t e = launch_pdl(engram::grad_w_reduce_kernel, blocks, (unsigned)engram::kReduceThreads,
                                     reinterpret_cast<cudaStream_t>(stream), w_partial, G,
                                     engram::reduce_groups(G), H,
                                     static_cast<const __nv_bfloat16 *>(wh),
                                     static_cast<const __nv_bfloat16 *>(we), dwh, dwe);
    if (e != cudaSuccess) return cuda_fail(e, "grad_w_reduce launch");
    return ENGRAM_OK;
}

// ---------------------------------------------------- gate bwd, fused reduce ----

engram_status_t engram_gate_bwd_fused(const void *grad_out, const void *x, const void *k,
                                      const void *v, const void *wh, const void *we, int64_t T,
                                      int32_t H, float eps, float scalar, void *dx, void *dk, void *dv,
                                      float *w_partial, int64_t G, uint32_t *tickets, float *dwh,
                                      float *dwe, engram_stream_t stream)
{
    engram_status_t st = check_gate_common(T, H, eps, scalar);
    if (st != ENGRAM_OK) return st;
    if (!wh || !we || !w_partial || !tickets || !dwh || !dwe)
        return fail(ENGRAM_ERR_INVALID_ARG, "wh, we, w_partial, tickets, dwh and dwe are required");
    if (T > 0 && (!grad_out || !x || !k || !v || !dx || !dk || !dv))
        return fail(ENGRAM_ERR_INVALID_ARG, "every tensor argument of engram_gate_bwd_fused is required");
    if (G < 1 || G > 0x7fffffff) return fail(ENGRAM_ERR_INVALID_ARG, "G=%lld not in [1, 2^31-1]", (long long)G);
    if (!aligned(grad_out, 2) || !aligned(x, 2) || !aligned(k, 2) || !aligned(v, 2) || !aligned(wh, 2) ||
        !aligned(we, 2) || !aligned(dx, 2) || !aligned(dk, 2) || !aligned(dv, 2))
        return fail(ENGRAM_ERR_INVALID_ARG, "bf16 tensors must be 2-byte aligned");
    if (!aligned(w_partial, 4) || !aligned(tickets, 4) || !aligned(dwh, 4) || !aligned(dwe, 4))
        return fail(ENGRAM_ERR_INVALID_ARG, "w_partial, tickets, dwh and dwe must be 4-byte aligned");
    if (!gate_tuned(H, {grad_out, x, k, v, wh, we, dx, dk, dv, w_partial})) {
        // generic shapes: the backward, then the standalone reduction (two launches)
        st = engram_gate_bwd(grad_out, x, k, v, wh, we, T, H, eps, scalar, dx, dk, dv, w_partial, G, stream);
        if (st != ENGRAM_OK) return st;
        return engram_grad_w_reduce(w_partial, G, H, wh, we, dwh, dwe, stream);
    }
    DeviceInfo dev;
    if ((st = device_info(&dev)) != ENGRAM_OK) return st;
    return launch_gate_bwd_tuned(dev, grad_out, x, k, v, wh, we, T, H, eps, scalar, dx, dk, dv, w_partial, G,
                                 tickets, dwh, dwe, reinterpret_cast<cudaStream_t>(stream));
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
    int64_t G = engram_gate_bwd_num_partials(T, H);
    if (G < 1) return ENGRAM_ERR_CUDA;  // message set by engram_gate_bwd_num_partials
    if ((size_t)H > kNoAllocPartialFloats)
        return fail(ENGRAM_ERR_UNSUPPORTED,
                    "engram_gate_bwd_noalloc: one partial row of H=%d floats exceeds its static scratch "
                    "of %zu floats", H, kNoAllocPartialFloats);
    // Fewer partial rows than recommended when they would not fit: the
    // backward's CTAs loop over tokens, so any G >= 1 gives the same gradients
    // (up to the order of the fp32 sums).
    G = std::min<int64_t>(G, (int64_t)(kNoAllocPartialFloats / (size_t)H));
    float *scratch = nullptr;
    if ((st = noalloc_scratch(&scratch)) != ENGRAM_OK) return st;
    // Every partial row the reduction reads is written by the backward first
    // (rows of CTAs without tokens as zeros), so nothing has to be cleared.
    st = engram_gate_bwd(grad_out, x, k, v, wh, we, T, H, eps, scalar, dx, dk, dv, scratch, G, stream);
    if (st != ENGRAM_OK) return st;
    return engram_grad_w_reduce(scratch, G, H, wh, we, dwh, dwe, stream);
}

// ------------------------------------------------------- gather backward ----

#include "gather_bwd_abi.inl"
