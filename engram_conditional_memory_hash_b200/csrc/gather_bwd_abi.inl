// C ABI of the Engram gather backward (engram_gather_bwd_workspace_size,
// engram_gather_bwd): workspace layout, argument checks and the launch
// sequence of the kernels in gather_bwd.cuh.  Included by engram_abi.cu,
// which provides fail(), aligned() and launch_pdl().

namespace {

constexpr int64_t kGbwdMaxEntries = int64_t(1) << 30;

// Offsets (bytes, 256-aligned) of the gather backward's scratch in the
// caller's workspace.  A region zeroed by every call first: the `seen` and
// `dupmap` bitmaps (one bit per table row) and the counters (list length,
// listed-chunk count).  Then the staging kernel's per-tile counts, two
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

// The list kernels (stage, sort, segments, carries) touch only the rows read
// more than once and the unique-row update only the others, so they run side
// by side: the list kernels on a side stream of the highest priority, forked
// from and joined back into the caller's stream with two events.  With the
// priority the list kernels' CTAs take the SM slots the update's short-lived
// CTAs free, ahead of the update's remaining CTAs.  One side stream and the
// two events per device, created on first use and kept until the process
// exits; the mutex is held while a call enqueues its work (the events are
// shared), so calls from several host threads take turns on the side stream.
struct GbwdFork {
    cudaStream_t side = nullptr;
    cudaEvent_t fork = nullptr, join = nullptr;
};
std::mutex g_gbwd_mutex;
GbwdFork g_gbwd_fork[kMaxDevices];

// With g_gbwd_mutex held.
engram_status_t gbwd_fork_objects(int dev, GbwdFork **out)
{
    GbwdFork &f = g_gbwd_fork[dev];
    if (f.side == nullptr) {
        int least = 0, greatest = 0;
        cudaError_t e = cudaDeviceGetStreamPriorityRange(&least, &greatest);
        if (e == cudaSuccess) e = cudaStreamCreateWithPriority(&f.side, cudaStreamNonBlocking, greatest);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&f.fork, cudaEventDisableTiming);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&f.join, cudaEventDisableTiming);
        if (e != cudaSuccess) return cuda_fail(e, "gather_bwd side stream");
    }
    *out = &f;
    return ENGRAM_OK;
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
    // the table of entry e is e mod LJ; its quotient by a reciprocal, exact for
    // every 32-bit e (the multiplier floor(2^64 / d) + 1, d < 2^32)
    p.lj_inv = p.LJ == 1 ? 0 : ~uint64_t(0) / (uint64_t)p.LJ + 1;
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

    DeviceInfo dev;
    if ((st = device_info(&dev)) != ENGRAM_OK) return st;
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
            (N + engram::kMarkThreads - 1) / engram::kMarkThreads, 16384);
        e = launch_pdl(engram::gbwd_mark_kernel, mblocks, (unsigned)engram::kMarkThreads, s, idx, p, seen,
                       dupmap);
    }
    if (e != cudaSuccess) return cuda_fail(e, "gather_bwd launch");
    // 2. fork: the list kernels (3-5) on the side stream, the unique-row
    //    update on the caller's stream, joined at the end
    std::lock_guard<std::mutex> fork_lock(g_gbwd_mutex);
    GbwdFork *fk = nullptr;
    if ((st = gbwd_fork_objects(dev.ordinal, &fk)) != ENGRAM_OK) return st;
    e = cudaEventRecord(fk->fork, s);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(fk->side, fk->fork, 0);
    if (e != cudaSuccess) return cuda_fail(e, "gather_bwd fork");
    cudaStream_t ls = fk->side;
    // the rows read once: updated in place on the caller's stream, one CTA per
    // tile of entries (short-lived CTAs, so that the list kernels find slots);
    // a programmatic dependent of the mark kernel, so that its first CTAs are
    // resident when the mark completes (145.8 against 147.4 us per call)
    {
        const unsigned ub = (unsigned)((N + engram::kUpdTile - 1) / engram::kUpdTile);
        const unsigned ut = (unsigned)engram::kUpdThreads;
        const uint32_t *dm = dupmap;
        auto uniq = [&](auto kern) { return launch_pdl(kern, ub, ut, s, idx, rows, p, dm, tab4); };
        e = nv <= 4 ? uniq(engram::gbwd_unique_kernel<4, 2>)
          : nv <= 8 ? uniq(engram::gbwd_unique_kernel<8, 2>)
          : nv <= 16 ? uniq(engram::gbwd_unique_kernel<16, 2>)
                     : uniq(engram::gbwd_unique_kernel<32, 2>);
    }
    // 3. the entries of rows read more than once, staged per tile (into the
    //    second buffer pair) with the first radix pass's tile histograms
    if (e == cudaSuccess) {
        engram::gbwd_stage_kernel<<<(unsigned)g.utiles, (unsigned)engram::kUniqThreads, 0, ls>>>(
            idx, p, static_cast<const uint32_t *>(dupmap), keys[1], vals[1], tile_cnt, hist, m_dev);
        e = cudaGetLastError();
    }
    // 4. stable radix sort by row of the staged entries into a contiguous
    //    list; keys lie in [0, R): sort on the bit length of R - 1
    int nbits = 0;
    while (nbits < 32 && (uint64_t(R - 1) >> nbits) != 0) ++nbits;
    const int npasses = std::max(1, (nbits + 7) / 8);
    const unsigned stiles = (unsigned)g.stiles, T_ = engram::kSortThreads;
    const uint32_t *no_cnt = nullptr;
    int cur = 1;   // the staged entries are in the second buffer pair
    // the first pass has one CTA per staged tile (all hold entries); the later
    // passes' grids, sized for a list of every entry, are capped at 4 CTAs per
    // SM looping over the list's tiles, so that fewer CTAs with nothing to do
    // compete with the update for SM slots (155.4 -> 152.1 us per call)
    const unsigned later = (unsigned)std::min<int64_t>(stiles, (int64_t)dev.sms * 4);
    for (int pass = 0; pass < npasses && e == cudaSuccess; ++pass) {
        const int shift = 8 * pass;
        if (pass > 0)
            e = launch_pdl(engram::gbwd_hist_kernel, later, T_, ls, static_cast<const uint32_t *>(keys[cur]), m_c,
                           shift, hist);
        if (e == cudaSuccess)
            e = launch_pdl(engram::gbwd_digit_scan_kernel, (unsigned)engram::kRadixBins,
                           (unsigned)engram::kScanThreads, ls, hist, m_c, pass == 0 ? g.utiles : int64_t(0),
                           totals);
        if (e == cudaSuccess)
            e = launch_pdl(engram::gbwd_scatter_kernel, pass == 0 ? (unsigned)g.utiles : later, T_, ls,
                           static_cast<const uint32_t *>(keys[cur]), static_cast<const uint32_t *>(vals[cur]),
                           m_c, pass == 0 ? static_cast<const uint32_t *>(tile_cnt) : no_cnt, shift,
                           static_cast<const uint32_t *>(hist), static_cast<const uint32_t *>(totals),
                           keys[1 - cur], vals[1 - cur], pass == 0 ? g.utiles : int64_t(0));
        cur = 1 - cur;
    }
    // 5. segments of the sorted list, then the segments that cross chunks
    const int64_t seg_blocks = (g.nchunks + engram::kSegThreads / 32 - 1) / (engram::kSegThreads / 32);
    // at most one wave of segment CTAs (4 per SM), looping over the chunks:
    // fewer CTAs that find nothing to do compete with the update for SM slots
    // (155.2 against 156.1 us per call; 2 per SM: 161.3)
    const unsigned blocks = (unsigned)std::min<int64_t>(seg_blocks, (int64_t)dev.sms * 4);
    const unsigned S_ = engram::kSegThreads;
    const uint32_t *kc = keys[cur], *vc = vals[cur];
    if (e == cudaSuccess) {
        if (nv <= 4)
            e = launch_pdl(engram::gbwd_segment_kernel<4, 1>, blocks, S_, ls, kc, vc, rows, p, tab4, carry_a,
                           carry_b, carry_list, carry_count, m_c);
        else if (nv <= 8)
            e = launch_pdl(engram::gbwd_segment_kernel<8, 1>, blocks, S_, ls, kc, vc, rows, p, tab4, carry_a,
                           carry_b, carry_list, carry_count, m_c);
        else if (nv <= 16)
            e = launch_pdl(engram::gbwd_segment_kernel<16, 1>, blocks, S_, ls, kc, vc, rows, p, tab4, carry_a,
                           carry_b, carry_list, carry_count, m_c);
        else
            e = launch_pdl(engram::gbwd_segment_kernel<32, 1>, blocks, S_, ls, kc, vc, rows, p, tab4, carry_a,
                           carry_b, carry_list, carry_count, m_c);
    }
    // one warp per listed chunk (a warp loops when more are listed than there
    // are warps: 8 per SM)
    const int64_t carry_warps = std::min<int64_t>(g.nchunks, (int64_t)dev.sms * 8);
    const unsigned carry_blocks = (unsigned)((carry_warps + engram::kCarryThreads / 32 - 1) /
                                             (engram::kCarryThreads / 32));
    const unsigned CT = engram::kCarryThreads;
    const double *ca = carry_a, *cb = carry_b;
    const uint32_t *cl = carry_list, *cn = carry_count;
    if (e == cudaSuccess) {
        auto carry = [&](auto kern) { return launch_pdl(kern, carry_blocks, CT, ls, kc, p, d_tables, ca, cb, cl, cn); };
        e = D <= 32 ? carry(engram::gbwd_carry_kernel<1>)
          : D <= 64 ? carry(engram::gbwd_carry_kernel<2>)
          : D <= 128 ? carry(engram::gbwd_carry_kernel<4>)
                     : carry(engram::gbwd_carry_kernel<8>);
    }
    // join: the caller's stream continues once the list kernels are done
    // (recorded even after a failed launch, so that the side stream never
    // runs ahead of a later call's fork)
    const cudaError_t ej = cudaEventRecord(fk->join, ls);
    const cudaError_t ew = ej == cudaSuccess ? cudaStreamWaitEvent(s, fk->join, 0) : ej;
    if (e == cudaSuccess) e = ew;
    if (e != cudaSuccess) return cuda_fail(e, "gather_bwd launch");
    return ENGRAM_OK;
}

}  // extern "C"
