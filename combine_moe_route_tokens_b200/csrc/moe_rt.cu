// moe_rt.cu — host side of libmoert.so: argument checks, launch
// configuration and the extern "C" entry points declared in moe_rt.h.
//
// Every entry point validates on the host, then enqueues its kernel(s) on the
// caller's stream and returns; nothing here synchronises with the device or
// reads device memory. The only host state is a per-device cache of
// attributes (SM count, shared-memory limit) with the kernel attribute setup,
// the programmatic-launch fallback flags and the NVTX switch.

#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstdio>
#include <atomic>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include <nvtx3/nvToolsExt.h>

#include "moe_rt.h"

#include "ptx.cuh"
#include "route.cuh"
#include "layout.cuh"
#include "dispatch.cuh"
#include "permute.cuh"
#include "combine.cuh"
#include "dedup.cuh"
#include "ep.cuh"

namespace {

using namespace moert;

constexpr uint64_t WAIT_LIMIT_NS = 1000000000ull;     // 1 s: every device-side wait gives up after this
constexpr uint64_t TEST_WAIT_LIMIT_NS = 10000000ull;  // 10 ms for MOE_FLAG_TEST_WAIT_TIMEOUT
constexpr size_t WS_TICKET_BYTES = 256; // layout workspaces: the ticket word, then the look-back words

using LayoutKernel = void (*)(LayoutArgs);
using DispatchKernel = void (*)(DispatchArgs);

LayoutKernel layout_count_for(int ipl)
{
    switch (ipl) {
    case 1:
        return layout_count_kernel<1>;
    case 2:
        return layout_count_kernel<2>;
    case 4:
        return layout_count_kernel<4>;
    case 8:
        return layout_count_kernel<8>;
    default:
        return layout_count_kernel<0>;
    }
}

LayoutKernel layout_fill_for(bool reroute, bool dense)
{
    if (reroute)
        return dense ? layout_fill_kernel<true, true> : layout_fill_kernel<true, false>;
    return dense ? layout_fill_kernel<false, true> : layout_fill_kernel<false, false>;
}

DispatchKernel dispatch_for(bool reroute, bool dense)
{
    if (reroute)
        return dense ? dispatch_kernel<true, true> : dispatch_kernel<true, false>;
    return dense ? dispatch_kernel<false, true> : dispatch_kernel<false, false>;
}

DispatchKernel dispatch_bulk_for(bool reroute, bool dense)
{
    if (reroute)
        return dense ? dispatch_bulk_kernel<true, true> : dispatch_bulk_kernel<true, false>;
    return dense ? dispatch_bulk_kernel<false, true> : dispatch_bulk_kernel<false, false>;
}

constexpr int LAYOUT_IPLS[] = {0, 1, 2, 4, 8};

// NVTX ranges around the enqueuing entry points, for profilers' timelines: on
// when the environment variable MOE_RT_NVTX is set to a non-empty value other
// than "0" (read once); off, a range costs one cached flag test.
bool nvtx_on()
{
    static const bool on = [] {
        const char *v = std::getenv("MOE_RT_NVTX");
        return v != nullptr && v[0] != '\0' && !(v[0] == '0' && v[1] == '\0');
    }();
    return on;
}

struct NvtxRange {
    const bool on;
    explicit NvtxRange(const char *name) : on(nvtx_on())
    {
        if (on)
            nvtxRangePushA(name);
    }
    ~NvtxRange()
    {
        if (on)
            nvtxRangePop();
    }
    NvtxRange(const NvtxRange &) = delete;
    NvtxRange &operator=(const NvtxRange &) = delete;
};

// Programmatic dependent launch is used unless the driver refuses it; then
// launches fall back to ordinary stream order.
std::atomic<bool> g_pdl_ok{true};

// Every kernel goes through cudaLaunchKernelEx with programmatic stream
// serialization, so its launch overlaps the tail of the previous kernel in the
// stream (each kernel calls pdl_wait() before reading anything a predecessor
// may have written).
template <typename... KArgs, typename... Args>
int launch(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, void *stream, Args... args)
{
    cudaLaunchAttribute attrs[1];
    unsigned n = 0;
    if (g_pdl_ok.load(std::memory_order_relaxed)) {
        attrs[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attrs[n].val.programmaticStreamSerializationAllowed = 1;
        ++n;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = static_cast<cudaStream_t>(stream);
    cfg.attrs = attrs;
    cfg.numAttrs = n;
    cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, args...);
    if (e != cudaSuccess && n > 0) {
        // retry without the programmatic attribute; only if that launch succeeds was the
        // attribute the cause, and only then is it dropped for later launches
        (void)cudaGetLastError();
        cfg.numAttrs = 0;
        e = cudaLaunchKernelEx(&cfg, kernel, args...);
        if (e == cudaSuccess)
            g_pdl_ok.store(false, std::memory_order_relaxed);
    }
    if (e != cudaSuccess) {
        (void)cudaGetLastError();
        return MOE_ERR_CUDA;
    }
    return MOE_OK;
}

struct DeviceInfo {
    int sms = 0;
    int smem_optin = 0;
    int layout_dyn_max = 0; // dynamic shared memory the layout kernels may take (opt-in limit less their static part)
    int tables_dyn_max = 0; // the same for the fill and fused dispatch kernels
    bool ready = false;
};

constexpr int MAX_DEVICES = 64;
DeviceInfo g_devices[MAX_DEVICES];
std::mutex g_mutex;

int device_info(DeviceInfo *out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= MAX_DEVICES)
        return MOE_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mutex);
    DeviceInfo &d = g_devices[dev];
    if (!d.ready) {
        if (cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&d.smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess)
            return MOE_ERR_CUDA;
        cudaError_t e = cudaSuccess;
        int static_max = 0;
        for (int ipl : LAYOUT_IPLS) {
            cudaFuncAttributes fa;
            if (e == cudaSuccess)
                e = cudaFuncGetAttributes(&fa, layout_count_for(ipl));
            if (e == cudaSuccess && static_cast<int>(fa.sharedSizeBytes) > static_max)
                static_max = static_cast<int>(fa.sharedSizeBytes);
        }
        d.layout_dyn_max = d.smem_optin - static_max;
        for (int ipl : LAYOUT_IPLS)
            if (e == cudaSuccess)
                e = cudaFuncSetAttribute(layout_count_for(ipl), cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         d.layout_dyn_max);
        // the second pass's per-CTA tables (at most ~57 KB for E_log = 2048 with as many replicas)
        int static2 = 0;
        for (int rr = 0; rr < 2; ++rr)
            for (int dn = 0; dn < 2; ++dn) {
                cudaFuncAttributes fa1, fa2;
                if (e == cudaSuccess)
                    e = cudaFuncGetAttributes(&fa1, layout_fill_for(rr != 0, dn != 0));
                if (e == cudaSuccess)
                    e = cudaFuncGetAttributes(&fa2, dispatch_for(rr != 0, dn != 0));
                cudaFuncAttributes fa3;
                if (e == cudaSuccess)
                    e = cudaFuncGetAttributes(&fa3, dispatch_bulk_for(rr != 0, dn != 0));
                if (e == cudaSuccess)
                    static2 = static_cast<int>(fa3.sharedSizeBytes) > static2 ? static_cast<int>(fa3.sharedSizeBytes)
                                                                             : static2;
                if (e == cudaSuccess) {
                    static2 = static_cast<int>(fa1.sharedSizeBytes) > static2 ? static_cast<int>(fa1.sharedSizeBytes)
                                                                             : static2;
                    static2 = static_cast<int>(fa2.sharedSizeBytes) > static2 ? static_cast<int>(fa2.sharedSizeBytes)
                                                                             : static2;
                }
            }
        d.tables_dyn_max = d.smem_optin - static2;
        for (int rr = 0; rr < 2; ++rr)
            for (int dn = 0; dn < 2; ++dn) {
                if (e == cudaSuccess)
                    e = cudaFuncSetAttribute(layout_fill_for(rr != 0, dn != 0),
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, d.tables_dyn_max);
                if (e == cudaSuccess)
                    e = cudaFuncSetAttribute(dispatch_for(rr != 0, dn != 0),
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, d.tables_dyn_max);
                if (e == cudaSuccess)
                    e = cudaFuncSetAttribute(dispatch_bulk_for(rr != 0, dn != 0),
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, d.tables_dyn_max);
            }
        if (e != cudaSuccess || d.layout_dyn_max <= 0)
            return MOE_ERR_CUDA;
        d.ready = true;
    }
    *out = d;
    return MOE_OK;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Derived sizes of a validated problem.
struct Dims {
    int64_t NK = 0;
    int64_t rows_max = 0;
    int32_t E = 0, E_loc = 0, M = 0, S = 0;
    int32_t A = 1; // row alignment
    int32_t T = 1; // TP folding peers
    int32_t C_local = 0;
};

int check_problem(const moe_problem_t *p, Dims *d)
{
    if (p == nullptr)
        return MOE_ERR_INVALID;
    if (p->N < 0 || p->H <= 0 || (p->H & 7) != 0 || p->k < 1 || p->E_log < 1 || p->R < 1 || p->capacity < 0 ||
        p->num_replicas < 0)
        return MOE_ERR_INVALID;
    if (p->E_log % p->R != 0 || p->num_replicas % p->R != 0 || p->num_replicas > p->E_log)
        return MOE_ERR_INVALID;
    if ((p->flags & ~(MOE_FLAG_TEST_WAIT_TIMEOUT | MOE_FLAG_DISPATCH_BULK_COPY)) != 0)
        return MOE_ERR_INVALID;
    if (p->row_align < 0 || p->tp_size < 0 || p->tp_rank < 0)
        return MOE_ERR_INVALID;
    const int64_t A = p->row_align > 1 ? p->row_align : 1;
    const int64_t T = p->tp_size > 1 ? p->tp_size : 1;
    if (T > MOE_MAX_TP || p->tp_rank >= T)
        return MOE_ERR_INVALID;
    const int64_t C_local = p->capacity > 0 ? (p->capacity + T - 1) / T : 0;
    if (p->capacity > 0 && C_local % A != 0)
        return MOE_ERR_INVALID;
    const int64_t NK = p->N * static_cast<int64_t>(p->k);
    if (p->N > (int64_t(1) << 40) || NK > INT32_MAX)
        return MOE_ERR_INVALID;
    const int64_t E = static_cast<int64_t>(p->E_log) + p->num_replicas;
    const int64_t rows_max = p->capacity > 0 ? E * C_local : (NK + E * (T - 1)) / T + E * (A - 1);
    if (rows_max > INT32_MAX)
        return MOE_ERR_INVALID;
    if (p->k > COMBINE_MAX_K || p->E_log > LAYOUT_MAX_E_LOG)
        return MOE_ERR_UNSUPPORTED;
    if (p->num_replicas > 0 && p->R > LAYOUT_MAX_PLACEMENT_RANKS)
        return MOE_ERR_UNSUPPORTED;
    if (static_cast<int64_t>(p->H) * 2 > INT32_MAX)
        return MOE_ERR_UNSUPPORTED;
    d->NK = NK;
    d->rows_max = rows_max;
    d->E = static_cast<int32_t>(E);
    d->E_loc = static_cast<int32_t>(E / p->R);
    d->M = p->E_log / p->R;
    d->S = p->num_replicas / p->R;
    d->A = static_cast<int32_t>(A);
    d->T = static_cast<int32_t>(T);
    d->C_local = static_cast<int32_t>(C_local);
    return MOE_OK;
}

// Per-assignment outputs may be NULL only when there are no assignments, per-row
// outputs only when there are no rows.
int check_layout(const moe_layout_t *l, const Dims &d, bool need_rows)
{
    if (l == nullptr || l->status == nullptr)
        return MOE_ERR_INVALID;
    if (d.NK > 0 && l->dest_row == nullptr)
        return MOE_ERR_INVALID;
    if (need_rows && d.rows_max > 0 && l->pad_mask == nullptr)
        return MOE_ERR_INVALID;
    return MOE_OK;
}

struct LayoutGrid {
    int32_t G;   // count blocks
    int32_t sub; // assignments per warp slice
    int32_t ipl; // assignments per lane kept in registers (1, 2, 4, 8), or 0 for longer slices
};

// The fewest ids per lane (1, 2, 4 or 8, in registers) that keep the count grid
// at LAYOUT_TARGET_BLOCKS blocks or fewer, so the look-back ends in one round;
// larger problems take 8 per lane on up to LAYOUT_MAX_BLOCKS blocks, and beyond
// that longer slices that are read twice.
LayoutGrid layout_grid(int64_t NK)
{
    const int64_t per_block_ipl1 = static_cast<int64_t>(LAYOUT_THREADS);
    int64_t ipl = 1;
    while (ipl < LAYOUT_MAX_IPL && (NK + per_block_ipl1 * ipl - 1) / (per_block_ipl1 * ipl) > LAYOUT_TARGET_BLOCKS)
        ipl <<= 1;
    int64_t G = (NK + per_block_ipl1 * ipl - 1) / (per_block_ipl1 * ipl);
    int32_t kind = static_cast<int32_t>(ipl);
    int64_t sub = 32 * ipl;
    if (G > LAYOUT_MAX_BLOCKS) { // slices longer than the registers hold
        kind = 0;
        const int64_t per_warp = (NK + static_cast<int64_t>(LAYOUT_MAX_BLOCKS) * LAYOUT_WARPS - 1) /
                                 (static_cast<int64_t>(LAYOUT_MAX_BLOCKS) * LAYOUT_WARPS);
        sub = ((per_warp + 31) / 32) * 32;
        G = (NK + LAYOUT_WARPS * sub - 1) / (LAYOUT_WARPS * sub);
    }
    if (G < 1)
        G = 1;
    return {static_cast<int32_t>(G), static_cast<int32_t>(sub), kind};
}

size_t layout_workspace_bytes(int32_t E_log)
{
    return WS_TICKET_BYTES + static_cast<size_t>(LAYOUT_MAX_BLOCKS) * static_cast<size_t>(E_log) * 8;
}

} // namespace

extern "C" {

int moe_abi_version(void) { return MOE_RT_ABI_VERSION; }

const char *moe_status_string(int code)
{
    switch (code) {
    case MOE_OK:
        return "ok";
    case MOE_ERR_INVALID:
        return "invalid argument (size, NULL pointer, alignment or inconsistent problem)";
    case MOE_ERR_UNSUPPORTED:
        return "valid problem beyond the kernels' limits";
    case MOE_ERR_CUDA:
        return "CUDA runtime call or kernel launch failed";
    case MOE_ERR_SCRATCH_LIMIT:
        return "problem needs more scratch than the library's fixed array holds (E_log above MOE_NOALLOC_MAX_E_LOG)";
    case static_cast<int>(MOE_DEV_EXPERT_RANGE):
        return "device: expert id outside [-1, E_log) skipped";
    case static_cast<int>(MOE_DEV_TIMEOUT):
        return "device: bounded wait ran out";
    case static_cast<int>(MOE_DEV_ROW_RANGE):
        return "device: destination row outside [-1, rows_max) skipped";
    default:
        return "unknown status";
    }
}

int64_t moe_rows_max(const moe_problem_t *problem)
{
    Dims d;
    const int rc = check_problem(problem, &d);
    return rc != MOE_OK ? rc : d.rows_max;
}

int moe_layout_workspace_bytes(const moe_problem_t *problem, size_t *bytes)
{
    Dims d;
    const int rc = check_problem(problem, &d);
    if (rc != MOE_OK)
        return rc;
    if (bytes == nullptr)
        return MOE_ERR_INVALID;
    *bytes = layout_workspace_bytes(problem->E_log);
    return MOE_OK;
}

int moe_route_topk(const float *logits, const uint8_t *token_mask, int64_t N, int32_t E, int32_t k,
                   int32_t *topk_idx, float *topk_probs, void *stream)
{
    NvtxRange nvtx_range("moe_route_topk");
    if (N < 0 || E < 1 || k < 1 || k > E)
        return MOE_ERR_INVALID;
    if (k > 32 || E > 1024)
        return MOE_ERR_UNSUPPORTED;
    if (N == 0)
        return MOE_OK;
    if (logits == nullptr || topk_idx == nullptr || topk_probs == nullptr)
        return MOE_ERR_INVALID;
    if (N > (int64_t(1) << 40))
        return MOE_ERR_INVALID;
    const int64_t blocks64 = (N + ROUTE_WARPS_PER_BLOCK - 1) / ROUTE_WARPS_PER_BLOCK;
    if (blocks64 > INT32_MAX)
        return MOE_ERR_UNSUPPORTED;
    const dim3 grid(static_cast<unsigned>(blocks64)), block(ROUTE_WARPS_PER_BLOCK * 32);
    const int vpl = (E + 31) / 32;
    auto go = [&](auto kernel) {
        return launch(kernel, grid, block, 0, stream, logits, token_mask, N, E, k, topk_idx, topk_probs);
    };
    if (vpl <= 1)
        return go(route_topk_kernel<1>);
    if (vpl <= 2)
        return go(route_topk_kernel<2>);
    if (vpl <= 4)
        return go(route_topk_kernel<4>);
    if (vpl <= 8)
        return go(route_topk_kernel<8>);
    if (vpl <= 16)
        return go(route_topk_kernel<16>);
    return go(route_topk_kernel<32>);
}

} // extern "C"

namespace {

// Host checks and arguments of the dispatch layout, shared by moe_dispatch_layout
// and moe_dispatch; nothing is enqueued.
int prepare_layout(const moe_problem_t *problem, const int32_t *topk_idx, const float *topk_probs,
                   const moe_layout_t *layout, void *workspace, size_t workspace_bytes, Dims &d, DeviceInfo &dev,
                   LayoutGrid &lg, LayoutArgs &a)
{
    int rc = check_problem(problem, &d);
    if (rc != MOE_OK)
        return rc;
    const moe_layout_t *l = layout;
    if (l == nullptr || l->status == nullptr || l->counts_logical == nullptr || l->placement == nullptr ||
        l->counts_raw == nullptr || l->tokens_per_expert == nullptr || l->expert_offsets == nullptr ||
        l->input_splits == nullptr || l->output_splits == nullptr || l->rank_offsets == nullptr ||
        l->counters == nullptr || l->num_rows == nullptr)
        return MOE_ERR_INVALID;
    if (d.NK > 0 && (topk_idx == nullptr || l->phys_idx == nullptr || l->ordinal == nullptr ||
                     l->dest_row == nullptr || l->drop_mask == nullptr))
        return MOE_ERR_INVALID;
    if (d.rows_max > 0 && (l->row_token == nullptr || l->row_slot == nullptr || l->row_local_expert == nullptr ||
                           l->row_prob == nullptr || l->pad_mask == nullptr))
        return MOE_ERR_INVALID;
    if (workspace == nullptr || workspace_bytes < layout_workspace_bytes(problem->E_log) ||
        (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
        return MOE_ERR_INVALID;
    if ((rc = device_info(&dev)) != MOE_OK)
        return rc;
    lg = layout_grid(d.NK);
    if (layout_count_smem_words(problem->E_log) * 4 > static_cast<size_t>(dev.layout_dyn_max) ||
        layout_tables_smem_words(problem->E_log, d.E) * 4 > static_cast<size_t>(dev.tables_dyn_max))
        return MOE_ERR_UNSUPPORTED;
    a.topk_idx = topk_idx;
    a.topk_probs = topk_probs;
    a.NK = d.NK;
    a.rows_max = d.rows_max;
    a.k = problem->k;
    a.E_log = problem->E_log;
    a.E = d.E;
    a.R = problem->R;
    a.E_loc = d.E_loc;
    a.M = d.M;
    a.S = d.S;
    a.num_replicas = problem->num_replicas;
    a.C = problem->capacity;
    a.A = d.A;
    a.T = d.T;
    a.tp_rank = problem->tp_rank;
    a.C_local = d.C_local;
    a.sub = lg.sub;
    a.G = lg.G;
    a.ws_ticket = static_cast<unsigned long long *>(workspace);
    a.ws_flags = reinterpret_cast<unsigned long long *>(static_cast<uint8_t *>(workspace) + WS_TICKET_BYTES);
    const bool test_timeout = (problem->flags & MOE_FLAG_TEST_WAIT_TIMEOUT) != 0;
    a.wait_limit_ns = test_timeout ? TEST_WAIT_LIMIT_NS : WAIT_LIMIT_NS;
    a.test_stall = test_timeout ? 1u : 0u;
    a.out = *l;
    return MOE_OK;
}

} // namespace

extern "C" {

int moe_dispatch_layout(const moe_problem_t *problem, const int32_t *topk_idx, const float *topk_probs,
                        const moe_layout_t *layout, void *workspace, size_t workspace_bytes, void *stream)
{
    NvtxRange nvtx_range("moe_dispatch_layout");
    Dims d;
    DeviceInfo dev;
    LayoutGrid lg;
    LayoutArgs a;
    int rc = prepare_layout(problem, topk_idx, topk_probs, layout, workspace, workspace_bytes, d, dev, lg, a);
    if (rc != MOE_OK)
        return rc;
    const int64_t fill_items = d.NK > d.rows_max ? d.NK : d.rows_max;
    const int64_t fill_blocks = fill_items > 0 ? (fill_items + FILL_THREADS - 1) / FILL_THREADS : 1;
    if (fill_blocks > INT32_MAX)
        return MOE_ERR_UNSUPPORTED;
    const bool reroute = problem->num_replicas > 0;
    const bool dense = problem->capacity == 0 && d.A == 1;
    rc = launch(layout_count_for(lg.ipl), dim3(lg.G), dim3(LAYOUT_THREADS), layout_count_smem_words(a.E_log) * 4, stream, a);
    if (rc != MOE_OK)
        return rc;
    return launch(layout_fill_for(reroute, dense), dim3(static_cast<unsigned>(fill_blocks)), dim3(FILL_THREADS),
                  layout_tables_smem_words(a.E_log, a.E) * 4, stream, a);
}

int moe_dispatch(const moe_problem_t *problem, const int32_t *topk_idx, const float *topk_probs,
                 const moe_layout_t *layout, void *workspace, size_t workspace_bytes, const uint16_t *hidden,
                 uint16_t *send, void *stream)
{
    NvtxRange nvtx_range("moe_dispatch");
    Dims d;
    DeviceInfo dev;
    LayoutGrid lg;
    DispatchArgs da;
    int rc = prepare_layout(problem, topk_idx, topk_probs, layout, workspace, workspace_bytes, d, dev, lg, da.L);
    if (rc != MOE_OK)
        return rc;
    if ((problem->N > 0 && (hidden == nullptr || !aligned16(hidden))) ||
        (d.rows_max > 0 && (send == nullptr || !aligned16(send))))
        return MOE_ERR_INVALID;
    da.hidden = reinterpret_cast<const uint4 *>(hidden);
    da.send = reinterpret_cast<uint4 *>(send);
    da.N = problem->N;
    da.V = problem->H / 8;
    const bool reroute = problem->num_replicas > 0;
    const bool dense = problem->capacity == 0 && d.A == 1;
    const size_t tables_bytes = layout_tables_smem_words(problem->E_log, d.E) * 4;
    DispatchKernel kernel;
    int64_t blocks;
    size_t smem;
    int threads;
    if ((problem->flags & MOE_FLAG_DISPATCH_BULK_COPY) == 0) {
        da.group = da.V <= 32 * PERMUTE_CHUNKS ? 32 : (da.V <= 64 * PERMUTE_CHUNKS ? 64 : PERMUTE_THREADS);
        da.pieces = (da.V + da.group * PERMUTE_CHUNKS - 1) / (da.group * PERMUTE_CHUNKS);
        const int64_t groups = PERMUTE_THREADS / da.group;
        threads = PERMUTE_THREADS;
        const int64_t rb = (d.rows_max + threads - 1) / threads; // row CTAs: at most four per SM; CTA 0 writes the tables
        da.row_ctas = static_cast<int32_t>(rb < 1 ? 1 : (rb < 4 * dev.sms ? rb : 4 * dev.sms));
        blocks = da.row_ctas + (problem->N * da.pieces + groups - 1) / groups;
        smem = tables_bytes;
        kernel = dispatch_for(reroute, dense);
    } else {
        // rows staged in shared memory: pieces of at most 32 KB; rows of at most 16 KB go several to a CTA
        const int64_t row_bytes = static_cast<int64_t>(da.V) * 16;
        da.pieces = static_cast<int32_t>((row_bytes + 32768 - 1) / 32768);
        da.group = da.pieces > 1 ? 1
                                 : static_cast<int32_t>(row_bytes >= 16384 ? 1
                                                                           : (16384 / row_bytes > TMA_MAX_TOKENS
                                                                                  ? TMA_MAX_TOKENS
                                                                                  : 16384 / row_bytes));
        threads = TMA_THREADS;
        const int64_t rb = (d.rows_max + threads - 1) / threads;
        da.row_ctas = static_cast<int32_t>(rb < 1 ? 1 : (rb < 4 * dev.sms ? rb : 4 * dev.sms));
        blocks = da.row_ctas + (da.pieces > 1 ? problem->N * da.pieces : (problem->N + da.group - 1) / da.group);
        const int64_t pchunks = (da.V + da.pieces - 1) / da.pieces;
        smem = ((tables_bytes / 4 + 31) & ~size_t(31)) * 4 + static_cast<size_t>(da.group) * pchunks * 16;
        if (smem > static_cast<size_t>(dev.tables_dyn_max))
            return MOE_ERR_UNSUPPORTED;
        kernel = dispatch_bulk_for(reroute, dense);
    }
    if (blocks > INT32_MAX)
        return MOE_ERR_UNSUPPORTED;
    rc = launch(layout_count_for(lg.ipl), dim3(lg.G), dim3(LAYOUT_THREADS),
                layout_count_smem_words(problem->E_log) * 4, stream, da.L);
    if (rc != MOE_OK)
        return rc;
    return launch(kernel, dim3(static_cast<unsigned>(blocks)), dim3(threads), smem, stream, da);
}

int moe_permute(const moe_problem_t *problem, const moe_layout_t *layout, const uint16_t *hidden, uint16_t *send,
                void *stream)
{
    NvtxRange nvtx_range("moe_permute");
    Dims d;
    int rc = check_problem(problem, &d);
    if (rc != MOE_OK)
        return rc;
    if ((rc = check_layout(layout, d, true)) != MOE_OK)
        return rc;
    if ((problem->N > 0 && (hidden == nullptr || !aligned16(hidden))) ||
        (d.rows_max > 0 && (send == nullptr || !aligned16(send))))
        return MOE_ERR_INVALID;
    if (problem->N == 0 && d.rows_max == 0)
        return MOE_OK;
    DeviceInfo dev;
    if ((rc = device_info(&dev)) != MOE_OK)
        return rc;

    PermuteArgs a;
    a.hidden = reinterpret_cast<const uint4 *>(hidden);
    a.send = reinterpret_cast<uint4 *>(send);
    a.dest_row = layout->dest_row;
    a.pad_mask = layout->pad_mask;
    a.status = layout->status;
    a.N = problem->N;
    a.rows_max = d.rows_max;
    a.k = problem->k;
    a.V = problem->H / 8;
    a.group = a.V <= 32 * PERMUTE_CHUNKS ? 32 : (a.V <= 64 * PERMUTE_CHUNKS ? 64 : PERMUTE_THREADS);
    a.pieces = (a.V + a.group * PERMUTE_CHUNKS - 1) / (a.group * PERMUTE_CHUNKS);
    a.load_first = problem->capacity == 0 ? 1 : 0;
    // pad-row workers: one warp checks 32 rows per pass, at most four CTAs per SM
    const int64_t zb = (d.rows_max + PERMUTE_THREADS - 1) / PERMUTE_THREADS;
    a.zero_blocks = static_cast<int32_t>(zb < 4 * dev.sms ? zb : 4 * dev.sms);
    const int64_t groups = PERMUTE_THREADS / a.group;
    const int64_t blocks = a.zero_blocks + (problem->N * a.pieces + groups - 1) / groups;
    if (blocks > INT32_MAX)
        return MOE_ERR_UNSUPPORTED;
    return launch(permute_kernel<false>, dim3(static_cast<unsigned>(blocks)), dim3(PERMUTE_THREADS), 0, stream, a);
}

namespace {

// Grid and launch for the combine kernel; `a` carries everything but the grid
// shape. SRC selects where slot rows are read: one buffer, TP peer buffers
// (restore) or EP receive buffers.
extern "C++" template <int SRC>
int launch_combine_args(CombineArgs a, int k, void *stream)
{
    if constexpr (SRC == SRC_LOCAL) {
        // short rows with one or two slots: several tokens per CTA, four chunks per thread
        if ((k == 1 || k == 2) && (a.V == 128 || a.V == 256 || a.V == 512 || a.V == 1024)) {
            const int64_t per_cta = COMBINE_THREADS / (a.V / COMBINE_ROW_CPT);
            int64_t blocks = (a.N + per_cta - 1) / per_cta;
            DeviceInfo dev;
            if (device_info(&dev) != MOE_OK)
                return MOE_ERR_CUDA;
            if (blocks > 4 * static_cast<int64_t>(dev.sms)) // grid-stride: four CTAs per SM (the register limit)
                blocks = 4 * static_cast<int64_t>(dev.sms);
            if (blocks > INT32_MAX)
                return MOE_ERR_UNSUPPORTED;
            const dim3 grid(static_cast<unsigned>(blocks)), block(COMBINE_THREADS);
            if (k == 1)
                return launch(combine_rows_kernel<1>, grid, block, 0, stream, a);
            return launch(combine_rows_kernel<2>, grid, block, 0, stream, a);
        }
    }
    // the widest CTA (up to 256 threads) that splits the row into equal parts
    const int v32 = ((a.V + 31) / 32) * 32;
    const int threads = v32 % 256 == 0 ? 256 : (v32 % 128 == 0 ? 128 : (v32 % 64 == 0 ? 64 : 32));
    a.nchunks = (a.V + threads - 1) / threads;
    const int64_t blocks = a.N * a.nchunks;
    if (blocks > INT32_MAX)
        return MOE_ERR_UNSUPPORTED;
    const dim3 grid(static_cast<unsigned>(blocks)), block(threads);
    switch (k) {
    case 1:
        return launch(combine_kernel<1, SRC>, grid, block, 0, stream, a);
    case 2:
        return launch(combine_kernel<2, SRC>, grid, block, 0, stream, a);
    case 4:
        return launch(combine_kernel<4, SRC>, grid, block, 0, stream, a);
    case 6:
        return launch(combine_kernel<6, SRC>, grid, block, 0, stream, a);
    case 8:
        return launch(combine_kernel<8, SRC>, grid, block, 0, stream, a);
    default:
        return launch(combine_kernel<0, SRC>, grid, block, 0, stream, a);
    }
}

int launch_combine(const moe_problem_t *problem, const moe_layout_t *layout, const uint16_t *y, const float *probs,
                   uint16_t *out, void *stream)
{
    Dims d;
    int rc = check_problem(problem, &d);
    if (rc != MOE_OK)
        return rc;
    if ((rc = check_layout(layout, d, false)) != MOE_OK)
        return rc;
    if (problem->N == 0)
        return MOE_OK;
    if (out == nullptr || !aligned16(out) || (d.rows_max > 0 && (y == nullptr || !aligned16(y))))
        return MOE_ERR_INVALID;
    CombineArgs a = {};
    a.y = reinterpret_cast<const uint4 *>(y);
    a.dest_row = layout->dest_row;
    a.probs = probs;
    a.out = reinterpret_cast<uint4 *>(out);
    a.status = layout->status;
    a.N = problem->N;
    a.rows_max = d.rows_max;
    a.k = problem->k;
    a.V = problem->H / 8;
    a.T = 1;
    a.last_first = 1; // right after a permute, its last rows are still in L2
    return launch_combine_args<SRC_LOCAL>(a, problem->k, stream);
}

} // namespace

int moe_combine(const moe_problem_t *problem, const moe_layout_t *layout, const uint16_t *expert_out,
                const float *topk_probs, uint16_t *out, void *stream)
{
    NvtxRange nvtx_range("moe_combine");
    return launch_combine(problem, layout, expert_out, topk_probs, out, stream);
}

int moe_permute_backward(const moe_problem_t *problem, const moe_layout_t *layout, const uint16_t *grad_send,
                         uint16_t *grad_hidden, void *stream)
{
    NvtxRange nvtx_range("moe_permute_backward");
    return launch_combine(problem, layout, grad_send, nullptr, grad_hidden, stream);
}

int moe_restore_combined(const moe_problem_t *problem, const moe_layout_t *peer_layouts,
                         const uint16_t *const *peer_expert_out, const float *topk_probs, uint16_t *out, void *stream)
{
    NvtxRange nvtx_range("moe_restore_combined");
    Dims d;
    int rc = check_problem(problem, &d);
    if (rc != MOE_OK)
        return rc;
    if (peer_layouts == nullptr || peer_expert_out == nullptr)
        return MOE_ERR_INVALID;
    for (int q = 0; q < d.T; ++q) {
        if ((rc = check_layout(&peer_layouts[q], d, false)) != MOE_OK)
            return rc;
        if (d.rows_max > 0 && (peer_expert_out[q] == nullptr || !aligned16(peer_expert_out[q])))
            return MOE_ERR_INVALID;
    }
    if (problem->N == 0)
        return MOE_OK;
    if (out == nullptr || !aligned16(out))
        return MOE_ERR_INVALID;
    CombineArgs a = {};
    a.probs = topk_probs;
    a.out = reinterpret_cast<uint4 *>(out);
    a.status = peer_layouts[0].status;
    a.N = problem->N;
    a.rows_max = d.rows_max;
    a.k = problem->k;
    a.V = problem->H / 8;
    a.T = d.T;
    for (int q = 0; q < d.T; ++q) {
        a.ys[q] = reinterpret_cast<const uint4 *>(peer_expert_out[q]);
        a.dests[q] = peer_layouts[q].dest_row;
    }
    a.last_first = 1;
    return launch_combine_args<SRC_TP_PEERS>(a, problem->k, stream);
}

int64_t moe_dedup_rows_max(const moe_problem_t *problem)
{
    Dims d;
    const int rc = check_problem(problem, &d);
    if (rc != MOE_OK)
        return rc;
    return problem->N * static_cast<int64_t>(problem->k < problem->R ? problem->k : problem->R);
}

int moe_dedup_workspace_bytes(const moe_problem_t *problem, size_t *bytes)
{
    Dims d;
    const int rc = check_problem(problem, &d);
    if (rc != MOE_OK)
        return rc;
    if (bytes == nullptr)
        return MOE_ERR_INVALID;
    *bytes = WS_TICKET_BYTES + static_cast<size_t>(DEDUP_MAX_BLOCKS) * problem->R * 8;
    return MOE_OK;
}

int moe_dedup_layout(const moe_problem_t *problem, const moe_layout_t *layout, const float *topk_probs,
                     const moe_dedup_t *dedup, void *workspace, size_t workspace_bytes, void *stream)
{
    NvtxRange nvtx_range("moe_dedup_layout");
    Dims d;
    int rc = check_problem(problem, &d);
    if (rc != MOE_OK)
        return rc;
    if (problem->R > MOE_MAX_DEDUP_RANKS)
        return MOE_ERR_UNSUPPORTED;
    const int64_t recv_max = moe_dedup_rows_max(problem);
    const moe_dedup_t *o = dedup;
    if (layout == nullptr || o == nullptr || o->status == nullptr || o->num_tokens_per_rank == nullptr ||
        o->recv_rank_offsets == nullptr || o->num_recv == nullptr)
        return MOE_ERR_INVALID;
    if (d.NK > 0 && (layout->phys_idx == nullptr || layout->dest_row == nullptr || o->is_token_in_rank == nullptr ||
                     o->token_rank_row == nullptr))
        return MOE_ERR_INVALID;
    if (recv_max > 0 && (o->recv_src_token == nullptr || o->recv_topk_idx == nullptr ||
                         o->recv_topk_weights == nullptr || o->recv_routing_map == nullptr ||
                         o->recv_probs == nullptr || o->recv_pad_mask == nullptr))
        return MOE_ERR_INVALID;
    if (recv_max > 0 && (d.E_loc & 3) == 0 &&
        (!aligned16(o->recv_probs) || (reinterpret_cast<uintptr_t>(o->recv_routing_map) & 3u) != 0))
        return MOE_ERR_INVALID;
    if (workspace == nullptr || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0 ||
        workspace_bytes < WS_TICKET_BYTES + static_cast<size_t>(DEDUP_MAX_BLOCKS) * problem->R * 8)
        return MOE_ERR_INVALID;
    int tpl = 1;
    while (tpl <= DEDUP_MAX_TPL &&
           (problem->N + static_cast<int64_t>(DEDUP_THREADS) * tpl - 1) / (static_cast<int64_t>(DEDUP_THREADS) * tpl) >
               DEDUP_MAX_BLOCKS)
        tpl <<= 1;
    if (tpl > DEDUP_MAX_TPL)
        return MOE_ERR_UNSUPPORTED;
    int64_t G = (problem->N + static_cast<int64_t>(DEDUP_THREADS) * tpl - 1) / (static_cast<int64_t>(DEDUP_THREADS) * tpl);
    if (G < 1)
        G = 1;
    const int64_t pairs = problem->N * problem->R;
    const int64_t fill_items = (pairs > recv_max ? pairs : recv_max) * DEDUP_FILL_LANES; // a group per pair and row
    const int64_t fill_blocks = fill_items > 0 ? (fill_items + DEDUP_FILL_THREADS - 1) / DEDUP_FILL_THREADS : 1;
    if (fill_blocks > INT32_MAX)
        return MOE_ERR_UNSUPPORTED;
    DedupArgs a;
    a.phys_idx = layout->phys_idx;
    a.dest_row = layout->dest_row;
    a.probs = topk_probs;
    a.N = problem->N;
    a.recv_max = recv_max;
    a.k = problem->k;
    a.R = problem->R;
    a.E_loc = d.E_loc;
    a.G = static_cast<int32_t>(G);
    a.ws_ticket = static_cast<unsigned long long *>(workspace);
    a.ws_flags = reinterpret_cast<unsigned long long *>(static_cast<uint8_t *>(workspace) + WS_TICKET_BYTES);
    a.wait_limit_ns = WAIT_LIMIT_NS;
    a.out = *o;
    const dim3 grid(static_cast<unsigned>(G)), block(DEDUP_THREADS);
    switch (tpl) {
    case 1:
        rc = launch(dedup_count_kernel<1>, grid, block, 0, stream, a);
        break;
    case 2:
        rc = launch(dedup_count_kernel<2>, grid, block, 0, stream, a);
        break;
    case 4:
        rc = launch(dedup_count_kernel<4>, grid, block, 0, stream, a);
        break;
    default:
        rc = launch(dedup_count_kernel<8>, grid, block, 0, stream, a);
        break;
    }
    if (rc != MOE_OK)
        return rc;
    DedupFillArgs f;
    f.phys_idx = layout->phys_idx;
    f.dest_row = layout->dest_row;
    f.probs = topk_probs;
    f.N = problem->N;
    f.recv_max = recv_max;
    f.k = problem->k;
    f.R = problem->R;
    f.E_loc = d.E_loc;
    f.G = a.G;
    f.ws_ticket = a.ws_ticket;
    f.ws_flags = a.ws_flags;
    f.out = *o;
    return launch(dedup_fill_kernel, dim3(static_cast<unsigned>(fill_blocks)), dim3(DEDUP_FILL_THREADS), 0, stream,
                  f);
}

int moe_dedup_dispatch(const moe_problem_t *problem, const moe_dedup_t *dedup, const uint16_t *hidden,
                       uint16_t *recv_x, void *stream)
{
    NvtxRange nvtx_range("moe_dedup_dispatch");
    Dims d;
    int rc = check_problem(problem, &d);
    if (rc != MOE_OK)
        return rc;
    if (problem->R > MOE_MAX_DEDUP_RANKS)
        return MOE_ERR_UNSUPPORTED;
    const int64_t recv_max = moe_dedup_rows_max(problem);
    if (dedup == nullptr || dedup->status == nullptr || (d.NK > 0 && dedup->token_rank_row == nullptr) ||
        (recv_max > 0 && dedup->recv_pad_mask == nullptr))
        return MOE_ERR_INVALID;
    if ((problem->N > 0 && (hidden == nullptr || !aligned16(hidden))) ||
        (recv_max > 0 && (recv_x == nullptr || !aligned16(recv_x))))
        return MOE_ERR_INVALID;
    if (recv_max == 0)
        return MOE_OK;
    DeviceInfo dev;
    if ((rc = device_info(&dev)) != MOE_OK)
        return rc;
    PermuteArgs a;
    a.hidden = reinterpret_cast<const uint4 *>(hidden);
    a.send = reinterpret_cast<uint4 *>(recv_x);
    a.dest_row = dedup->token_rank_row;
    a.pad_mask = dedup->recv_pad_mask;
    a.status = dedup->status;
    a.N = problem->N;
    a.rows_max = recv_max;
    a.k = problem->R;
    a.V = problem->H / 8;
    a.group = a.V <= 32 * PERMUTE_CHUNKS ? 32 : (a.V <= 64 * PERMUTE_CHUNKS ? 64 : PERMUTE_THREADS);
    a.pieces = (a.V + a.group * PERMUTE_CHUNKS - 1) / (a.group * PERMUTE_CHUNKS);
    a.load_first = problem->capacity == 0 ? 1 : 0;
    const int64_t zb = (recv_max + PERMUTE_THREADS - 1) / PERMUTE_THREADS;
    a.zero_blocks = static_cast<int32_t>(zb < 4 * dev.sms ? zb : 4 * dev.sms);
    const int64_t groups = PERMUTE_THREADS / a.group;
    const int64_t blocks = a.zero_blocks + (problem->N * a.pieces + groups - 1) / groups;
    if (blocks > INT32_MAX)
        return MOE_ERR_UNSUPPORTED;
    return launch(permute_kernel<false>, dim3(static_cast<unsigned>(blocks)), dim3(PERMUTE_THREADS), 0, stream, a);
}

int moe_dedup_combine_local(const moe_problem_t *problem, const moe_layout_t *layout, const moe_dedup_t *dedup,
                            const uint16_t *expert_out, const float *topk_probs, uint16_t *partial, void *stream)
{
    NvtxRange nvtx_range("moe_dedup_combine_local");
    Dims d;
    int rc = check_problem(problem, &d);
    if (rc != MOE_OK)
        return rc;
    if (problem->R > MOE_MAX_DEDUP_RANKS)
        return MOE_ERR_UNSUPPORTED;
    const int64_t recv_max = moe_dedup_rows_max(problem);
    if ((rc = check_layout(layout, d, false)) != MOE_OK)
        return rc;
    if (layout->rank_offsets == nullptr || dedup == nullptr || dedup->status == nullptr ||
        dedup->num_recv == nullptr || (d.NK > 0 && dedup->token_rank_row == nullptr))
        return MOE_ERR_INVALID;
    if ((d.rows_max > 0 && (expert_out == nullptr || !aligned16(expert_out))) ||
        (recv_max > 0 && (partial == nullptr || !aligned16(partial))))
        return MOE_ERR_INVALID;
    if (recv_max == 0)
        return MOE_OK;
    DedupCombineArgs a;
    a.y = reinterpret_cast<const uint4 *>(expert_out);
    a.dest_row = layout->dest_row;
    a.probs = topk_probs;
    a.rank_offsets = layout->rank_offsets;
    a.token_rank_row = dedup->token_rank_row;
    a.partial = reinterpret_cast<uint4 *>(partial);
    a.status = dedup->status;
    a.N = problem->N;
    a.recv_max = recv_max;
    a.rows_max = d.rows_max;
    a.k = problem->k;
    a.R = problem->R;
    a.V = problem->H / 8;
    // token-major, as the combine: the widest CTA (up to 256 threads) that splits the row into equal parts
    const int v32 = ((a.V + 31) / 32) * 32;
    const int threads = v32 % 256 == 0 ? 256 : (v32 % 128 == 0 ? 128 : (v32 % 64 == 0 ? 64 : 32));
    a.nchunks = (a.V + threads - 1) / threads;
    a.num_recv = dedup->num_recv;
    a.token_blocks = problem->N * a.nchunks;
    // trailing CTAs zero the receive rows past num_recv (a count known on the device only)
    DeviceInfo dev;
    if ((rc = device_info(&dev)) != MOE_OK)
        return rc;
    const int64_t tail_work = (recv_max * a.V + threads - 1) / threads;
    const int64_t zero_blocks = tail_work < 2 * dev.sms ? tail_work : 2 * dev.sms;
    const int64_t blocks = a.token_blocks + zero_blocks;
    if (blocks > INT32_MAX)
        return MOE_ERR_UNSUPPORTED;
    const dim3 grid(static_cast<unsigned>(blocks)), block(threads);
    switch (problem->k) {
    case 1:
        return launch(dedup_combine_local_kernel<1>, grid, block, 0, stream, a);
    case 2:
        return launch(dedup_combine_local_kernel<2>, grid, block, 0, stream, a);
    case 4:
        return launch(dedup_combine_local_kernel<4>, grid, block, 0, stream, a);
    case 6:
        return launch(dedup_combine_local_kernel<6>, grid, block, 0, stream, a);
    case 8:
        return launch(dedup_combine_local_kernel<8>, grid, block, 0, stream, a);
    default:
        return launch(dedup_combine_local_kernel<0>, grid, block, 0, stream, a);
    }
}

int moe_dedup_combine(const moe_problem_t *problem, const moe_dedup_t *dedup, const uint16_t *partial,
                      uint16_t *out, void *stream)
{
    NvtxRange nvtx_range("moe_dedup_combine");
    Dims d;
    int rc = check_problem(problem, &d);
    if (rc != MOE_OK)
        return rc;
    if (problem->R > MOE_MAX_DEDUP_RANKS)
        return MOE_ERR_UNSUPPORTED;
    const int64_t recv_max = moe_dedup_rows_max(problem);
    if (dedup == nullptr || dedup->status == nullptr || (d.NK > 0 && dedup->token_rank_row == nullptr))
        return MOE_ERR_INVALID;
    if (problem->N == 0)
        return MOE_OK;
    if (out == nullptr || !aligned16(out) || (recv_max > 0 && (partial == nullptr || !aligned16(partial))))
        return MOE_ERR_INVALID;
    CombineArgs a = {};
    a.y = reinterpret_cast<const uint4 *>(partial);
    a.dest_row = dedup->token_rank_row;
    a.probs = nullptr; // unit weights: the partials are already weighted
    a.out = reinterpret_cast<uint4 *>(out);
    a.status = dedup->status;
    a.N = problem->N;
    a.rows_max = recv_max;
    a.k = problem->R;
    a.V = problem->H / 8;
    a.T = 1;
    a.last_first = 0; // the receiver pass wrote its partials last first: read them first first
    return launch_combine_args<SRC_LOCAL>(a, problem->R, stream);
}

int64_t moe_ep_recv_rows_max(const moe_problem_t *problem)
{
    Dims d;
    const int rc = check_problem(problem, &d);
    if (rc != MOE_OK)
        return rc;
    if (d.T != 1 || problem->R > MOE_MAX_EP_RANKS)
        return MOE_ERR_UNSUPPORTED;
    // rows one source can send to one rank, times the sources
    int64_t per = problem->capacity > 0 ? static_cast<int64_t>(d.E_loc) * d.C_local
                                        : d.NK + static_cast<int64_t>(d.E_loc) * (d.A - 1);
    if (per > d.rows_max)
        per = d.rows_max;
    return per * problem->R;
}

int moe_ep_plan(const moe_problem_t *problem, const int32_t *offsets_all, int32_t src_rank, int32_t *base,
                int32_t *recv_expert_offsets, int32_t *num_recv, uint32_t *status, void *stream)
{
    NvtxRange nvtx_range("moe_ep_plan");
    Dims d;
    int rc = check_problem(problem, &d);
    if (rc != MOE_OK)
        return rc;
    const int64_t recv_max = moe_ep_recv_rows_max(problem);
    if (recv_max < 0)
        return static_cast<int>(recv_max);
    if (d.E > EP_PLAN_THREADS * EP_PLAN_PER)
        return MOE_ERR_UNSUPPORTED;
    if (src_rank < 0 || src_rank >= problem->R || offsets_all == nullptr || base == nullptr ||
        recv_expert_offsets == nullptr || num_recv == nullptr || status == nullptr)
        return MOE_ERR_INVALID;
    if (recv_max > INT32_MAX)
        return MOE_ERR_UNSUPPORTED;
    EpPlanArgs a;
    a.offsets_all = offsets_all;
    a.R = problem->R;
    a.E = d.E;
    a.E_loc = d.E_loc;
    a.src = src_rank;
    a.recv_max = recv_max;
    a.base = base;
    a.recv_expert_offsets = recv_expert_offsets;
    a.num_recv = num_recv;
    a.status = status;
    const size_t smem = (2 * static_cast<size_t>(d.E) + 1) * sizeof(int32_t);
    return launch(ep_plan_kernel, dim3(1), dim3(EP_PLAN_THREADS), smem, stream, a);
}

int moe_ep_publish_offsets(const moe_problem_t *problem, const int32_t *expert_offsets, int32_t src_rank,
                           int32_t *const *peer_offsets_tables, void *stream)
{
    NvtxRange nvtx_range("moe_ep_publish_offsets");
    Dims d;
    int rc = check_problem(problem, &d);
    if (rc != MOE_OK)
        return rc;
    if (problem->tp_size > 1 || problem->R > MOE_MAX_EP_RANKS)
        return MOE_ERR_UNSUPPORTED;
    if (src_rank < 0 || src_rank >= problem->R || expert_offsets == nullptr || peer_offsets_tables == nullptr)
        return MOE_ERR_INVALID;
    EpPublishArgs a;
    a.offsets = expert_offsets;
    a.peer_tables = peer_offsets_tables;
    a.R = problem->R;
    a.E = d.E;
    a.src = src_rank;
    const int64_t n = static_cast<int64_t>(a.R) * (a.E + 1);
    const int64_t blocks = (n + 255) / 256;
    return launch(ep_publish_offsets_kernel, dim3(static_cast<unsigned>(blocks < 64 ? blocks : 64)), dim3(256), 0, stream, a);
}

int moe_ep_dispatch(const moe_problem_t *problem, const moe_layout_t *layout, const int32_t *base,
                    const uint16_t *hidden, uint16_t *const *peer_recv, void *stream)
{
    NvtxRange nvtx_range("moe_ep_dispatch");
    Dims d;
    int rc = check_problem(problem, &d);
    if (rc != MOE_OK)
        return rc;
    const int64_t recv_max = moe_ep_recv_rows_max(problem);
    if (recv_max < 0)
        return static_cast<int>(recv_max);
    if ((rc = check_layout(layout, d, false)) != MOE_OK)
        return rc;
    if (layout->expert_offsets == nullptr || layout->tokens_per_expert == nullptr || base == nullptr ||
        peer_recv == nullptr || (d.NK > 0 && layout->phys_idx == nullptr))
        return MOE_ERR_INVALID;
    if (problem->N > 0 && (hidden == nullptr || !aligned16(hidden)))
        return MOE_ERR_INVALID;
    if (problem->N == 0)
        return MOE_OK;
    DeviceInfo dev;
    if ((rc = device_info(&dev)) != MOE_OK)
        return rc;
    PermuteArgs a = {};
    a.hidden = reinterpret_cast<const uint4 *>(hidden);
    a.dest_row = layout->dest_row;
    a.status = layout->status;
    a.N = problem->N;
    a.rows_max = d.rows_max;
    a.k = problem->k;
    a.V = problem->H / 8;
    a.group = a.V <= 32 * PERMUTE_CHUNKS ? 32 : (a.V <= 64 * PERMUTE_CHUNKS ? 64 : PERMUTE_THREADS);
    a.pieces = (a.V + a.group * PERMUTE_CHUNKS - 1) / (a.group * PERMUTE_CHUNKS);
    a.load_first = problem->capacity == 0 ? 1 : 0;
    a.ep_peers = reinterpret_cast<uint4 *const *>(peer_recv);
    a.phys_idx = layout->phys_idx;
    a.ep_base = base;
    a.ep_offsets = layout->expert_offsets;
    a.ep_tokens = layout->tokens_per_expert;
    a.recv_max = recv_max;
    a.E = d.E;
    a.E_loc = d.E_loc;
    // padding rows exist only with a capacity or a row alignment: one warp per expert
    const bool pads = problem->capacity > 0 || d.A > 1;
    const int64_t zb = pads ? (d.E + PERMUTE_THREADS / 32 - 1) / (PERMUTE_THREADS / 32) : 0;
    a.zero_blocks = static_cast<int32_t>(zb < 4 * dev.sms ? zb : 4 * dev.sms);
    const int64_t groups = PERMUTE_THREADS / a.group;
    const int64_t blocks = a.zero_blocks + (problem->N * a.pieces + groups - 1) / groups;
    if (blocks > INT32_MAX)
        return MOE_ERR_UNSUPPORTED;
    return launch(permute_kernel<true>, dim3(static_cast<unsigned>(blocks)), dim3(PERMUTE_THREADS), 0, stream, a);
}

int moe_ep_combine(const moe_problem_t *problem, const moe_layout_t *layout, const int32_t *base,
                   const uint16_t *const *peer_expert_out, const float *topk_probs, uint16_t *out, void *stream)
{
    NvtxRange nvtx_range("moe_ep_combine");
    Dims d;
    int rc = check_problem(problem, &d);
    if (rc != MOE_OK)
        return rc;
    const int64_t recv_max = moe_ep_recv_rows_max(problem);
    if (recv_max < 0)
        return static_cast<int>(recv_max);
    if ((rc = check_layout(layout, d, false)) != MOE_OK)
        return rc;
    if (layout->expert_offsets == nullptr || base == nullptr || peer_expert_out == nullptr ||
        (d.NK > 0 && layout->phys_idx == nullptr))
        return MOE_ERR_INVALID;
    if (problem->N == 0)
        return MOE_OK;
    if (out == nullptr || !aligned16(out))
        return MOE_ERR_INVALID;
    CombineArgs a = {};
    a.dest_row = layout->dest_row;
    a.probs = topk_probs;
    a.out = reinterpret_cast<uint4 *>(out);
    a.status = layout->status;
    a.N = problem->N;
    a.rows_max = d.rows_max;
    a.k = problem->k;
    a.V = problem->H / 8;
    a.T = 1;
    a.ep_peers = reinterpret_cast<const uint4 *const *>(peer_expert_out);
    a.phys_idx = layout->phys_idx;
    a.ep_base = base;
    a.ep_offsets = layout->expert_offsets;
    a.recv_max = recv_max;
    a.E = d.E;
    a.E_loc = d.E_loc;
    a.last_first = 1;
    return launch_combine_args<SRC_EP>(a, problem->k, stream);
}

int moe_ep_combine_backward(const moe_problem_t *problem, const moe_layout_t *layout, const int32_t *base,
                            const uint16_t *grad_out, const uint16_t *const *peer_expert_out, const float *topk_probs,
                            uint16_t *const *peer_grad_expert_out, float *grad_probs, void *stream)
{
    NvtxRange nvtx_range("moe_ep_combine_backward");
    Dims d;
    int rc = check_problem(problem, &d);
    if (rc != MOE_OK)
        return rc;
    const int64_t recv_max = moe_ep_recv_rows_max(problem);
    if (recv_max < 0)
        return static_cast<int>(recv_max);
    if ((rc = check_layout(layout, d, false)) != MOE_OK)
        return rc;
    if (layout->expert_offsets == nullptr || layout->tokens_per_expert == nullptr || base == nullptr ||
        peer_expert_out == nullptr || peer_grad_expert_out == nullptr || (d.NK > 0 && layout->phys_idx == nullptr))
        return MOE_ERR_INVALID;
    if (problem->N == 0)
        return MOE_OK;
    if (grad_out == nullptr || !aligned16(grad_out) || topk_probs == nullptr || grad_probs == nullptr)
        return MOE_ERR_INVALID;
    DeviceInfo dev;
    if ((rc = device_info(&dev)) != MOE_OK)
        return rc;
    CombineBwdArgs a = {};
    a.grad_out = reinterpret_cast<const uint4 *>(grad_out);
    a.dest_row = layout->dest_row;
    a.probs = topk_probs;
    a.grad_probs = grad_probs;
    a.status = layout->status;
    a.N = problem->N;
    a.rows_max = d.rows_max;
    a.k = problem->k;
    a.V = problem->H / 8;
    a.ep_peer_y = reinterpret_cast<const uint4 *const *>(peer_expert_out);
    a.ep_peer_gy = reinterpret_cast<uint4 *const *>(peer_grad_expert_out);
    a.phys_idx = layout->phys_idx;
    a.ep_base = base;
    a.ep_offsets = layout->expert_offsets;
    a.ep_tokens = layout->tokens_per_expert;
    a.recv_max = recv_max;
    a.E = d.E;
    a.E_loc = d.E_loc;
    a.R = problem->R;
    // this rank's padding rows in the owners' gradient buffers: one warp per expert
    const bool pads = problem->capacity > 0 || d.A > 1;
    const int64_t zb = pads ? (d.E + COMBINE_BWD_THREADS / 32 - 1) / (COMBINE_BWD_THREADS / 32) : 0;
    a.zero_blocks = static_cast<int32_t>(zb < 2 * dev.sms ? zb : 2 * dev.sms);
    const int64_t blocks = problem->N + a.zero_blocks;
    if (blocks > INT32_MAX)
        return MOE_ERR_UNSUPPORTED;
    const dim3 grid(static_cast<unsigned>(blocks)), block(COMBINE_BWD_THREADS);
    switch (problem->k) {
    case 1:
        return launch(combine_backward_kernel<1, true>, grid, block, 0, stream, a);
    case 2:
        return launch(combine_backward_kernel<2, true>, grid, block, 0, stream, a);
    case 4:
        return launch(combine_backward_kernel<4, true>, grid, block, 0, stream, a);
    case 6:
        return launch(combine_backward_kernel<6, true>, grid, block, 0, stream, a);
    case 8:
        return launch(combine_backward_kernel<8, true>, grid, block, 0, stream, a);
    default:
        return launch(combine_backward_kernel<0, true>, grid, block, 0, stream, a);
    }
}

int moe_combine_backward(const moe_problem_t *problem, const moe_layout_t *layout, const uint16_t *grad_out,
                         const uint16_t *expert_out, const float *topk_probs, uint16_t *grad_expert_out,
                         float *grad_probs, void *stream)
{
    NvtxRange nvtx_range("moe_combine_backward");
    Dims d;
    int rc = check_problem(problem, &d);
    if (rc != MOE_OK)
        return rc;
    if ((rc = check_layout(layout, d, true)) != MOE_OK)
        return rc;
    if (problem->N > 0 && (grad_out == nullptr || !aligned16(grad_out) || topk_probs == nullptr ||
                           grad_probs == nullptr))
        return MOE_ERR_INVALID;
    if (d.rows_max > 0 && (expert_out == nullptr || !aligned16(expert_out) || grad_expert_out == nullptr ||
                           !aligned16(grad_expert_out)))
        return MOE_ERR_INVALID;
    if (problem->N == 0 && d.rows_max == 0)
        return MOE_OK;
    DeviceInfo dev;
    if ((rc = device_info(&dev)) != MOE_OK)
        return rc;
    CombineBwdArgs a = {};
    a.grad_out = reinterpret_cast<const uint4 *>(grad_out);
    a.y = reinterpret_cast<const uint4 *>(expert_out);
    a.dest_row = layout->dest_row;
    a.probs = topk_probs;
    a.pad_mask = layout->pad_mask;
    a.grad_y = reinterpret_cast<uint4 *>(grad_expert_out);
    a.grad_probs = grad_probs;
    a.status = layout->status;
    a.N = problem->N;
    a.rows_max = d.rows_max;
    a.k = problem->k;
    a.V = problem->H / 8;
    int64_t zb = (d.rows_max + 63) / 64;
    const int64_t zmax = static_cast<int64_t>(dev.sms) * 2;
    a.zero_blocks = static_cast<int32_t>(zb > zmax ? zmax : zb);
    const int64_t blocks = problem->N + a.zero_blocks;
    if (blocks > INT32_MAX)
        return MOE_ERR_UNSUPPORTED;
    const dim3 grid(static_cast<unsigned>(blocks)), block(COMBINE_BWD_THREADS);
    switch (problem->k) {
    case 1:
        return launch(combine_backward_kernel<1>, grid, block, 0, stream, a);
    case 2:
        return launch(combine_backward_kernel<2>, grid, block, 0, stream, a);
    case 4:
        return launch(combine_backward_kernel<4>, grid, block, 0, stream, a);
    case 6:
        return launch(combine_backward_kernel<6>, grid, block, 0, stream, a);
    case 8:
        return launch(combine_backward_kernel<8>, grid, block, 0, stream, a);
    default:
        return launch(combine_backward_kernel<0>, grid, block, 0, stream, a);
    }
}

} // extern "C"

// ------------------------------------------------ layout without allocation --
// moe_dispatch_layout_noalloc: the same layout, with its scratch in a
// fixed device array of this library instead of a caller-provided workspace,
// for callers that cannot allocate device memory.

namespace {

static_assert(MOE_NOALLOC_SCRATCH_BYTES ==
                  WS_TICKET_BYTES + static_cast<size_t>(LAYOUT_MAX_BLOCKS) * MOE_NOALLOC_MAX_E_LOG * 8,
              "fixed scratch must hold the ticket word and LAYOUT_MAX_BLOCKS rows of look-back words");

// Held by every device that loads the library, for the life of the process.
static __device__ __align__(256) unsigned char g_layout_scratch[MOE_NOALLOC_SCRATCH_BYTES];

struct ScratchAddress {
    void *ptr = nullptr;
    bool ready = false;
};
ScratchAddress g_scratch_address[MAX_DEVICES];
std::mutex g_scratch_mutex;

// Device address of g_layout_scratch on device `dev`, looked up once per device
// with that device current (in host code the symbol is only a stand-in, not a
// device address).
int scratch_address(int dev, void **out)
{
    if (dev < 0 || dev >= MAX_DEVICES)
        return MOE_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    ScratchAddress &s = g_scratch_address[dev];
    if (!s.ready) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_layout_scratch) != cudaSuccess || p == nullptr) {
            (void)cudaGetLastError();
            return MOE_ERR_CUDA;
        }
        s.ptr = p;
        s.ready = true;
    }
    *out = s.ptr;
    return MOE_OK;
}

} // namespace

extern "C" int moe_dispatch_layout_noalloc(const moe_problem_t *problem, const int32_t *topk_idx,
                                           const float *topk_probs, const moe_layout_t *layout, void *stream)
{
    NvtxRange nvtx_range("moe_dispatch_layout_noalloc");
    Dims d;
    int rc = check_problem(problem, &d);
    if (rc != MOE_OK)
        return rc;
    if (problem->E_log > MOE_NOALLOC_MAX_E_LOG)
        return MOE_ERR_SCRATCH_LIMIT;
    // the argument checks of moe_dispatch_layout, made before anything is enqueued here
    const moe_layout_t *l = layout;
    if (l == nullptr || l->status == nullptr || l->counts_logical == nullptr || l->placement == nullptr ||
        l->counts_raw == nullptr || l->tokens_per_expert == nullptr || l->expert_offsets == nullptr ||
        l->input_splits == nullptr || l->output_splits == nullptr || l->rank_offsets == nullptr ||
        l->counters == nullptr || l->num_rows == nullptr)
        return MOE_ERR_INVALID;
    if (d.NK > 0 && (topk_idx == nullptr || l->phys_idx == nullptr || l->ordinal == nullptr ||
                     l->dest_row == nullptr || l->drop_mask == nullptr))
        return MOE_ERR_INVALID;
    if (d.rows_max > 0 && (l->row_token == nullptr || l->row_slot == nullptr || l->row_local_expert == nullptr ||
                           l->row_prob == nullptr || l->pad_mask == nullptr))
        return MOE_ERR_INVALID;
    // The scratch must be the array of the device that runs the call: the one that
    // owns `stream`. Kernels launch on the current device, so the two must agree.
    int cur = 0, owner = 0;
    if (cudaGetDevice(&cur) != cudaSuccess || cudaStreamGetDevice(static_cast<cudaStream_t>(stream), &owner) !=
                                                   cudaSuccess) {
        (void)cudaGetLastError();
        return MOE_ERR_CUDA;
    }
    if (owner != cur)
        return MOE_ERR_INVALID;
    void *scratch = nullptr;
    if ((rc = scratch_address(cur, &scratch)) != MOE_OK)
        return rc;
    // Nothing in the array has to be cleared between calls: every look-back word
    // carries the epoch of the launch that wrote it, and the ticket word is
    // rolled over by the last block of each launch (also after a timed-out one).
    return moe_dispatch_layout(problem, topk_idx, topk_probs, layout, scratch, MOE_NOALLOC_SCRATCH_BYTES, stream);
}

// ------------------------------------------------------------- CUDA IPC --
// Sharing a buffer between processes of the expert-parallel exchange: the
// allocation that holds it is exported with cudaIpcGetMemHandle together with
// the buffer's offset inside it (a caching allocator hands out pieces of larger
// allocations); a peer maps the allocation with cudaIpcOpenMemHandle.

namespace {

using AddressRangeFn = CUresult (*)(CUdeviceptr *, size_t *, CUdeviceptr);

AddressRangeFn address_range_fn()
{
    static AddressRangeFn fn = [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuMemGetAddressRange", &p, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess) {
            (void)cudaGetLastError();
            return static_cast<AddressRangeFn>(nullptr);
        }
        return reinterpret_cast<AddressRangeFn>(p);
    }();
    return fn;
}

static_assert(sizeof(cudaIpcMemHandle_t) == sizeof(((moe_ipc_buffer_t *)nullptr)->handle),
              "moe_ipc_buffer_t.handle must hold a cudaIpcMemHandle_t");

} // namespace

extern "C" int moe_ipc_export(const void *ptr, size_t bytes, moe_ipc_buffer_t *out)
{
    if (ptr == nullptr || out == nullptr)
        return MOE_ERR_INVALID;
    AddressRangeFn range = address_range_fn();
    if (range == nullptr)
        return MOE_ERR_CUDA;
    CUdeviceptr base = 0;
    size_t size = 0;
    if (range(&base, &size, reinterpret_cast<CUdeviceptr>(ptr)) != CUDA_SUCCESS)
        return MOE_ERR_INVALID; // not device memory of this process
    const uint64_t offset = reinterpret_cast<uint64_t>(ptr) - static_cast<uint64_t>(base);
    if (offset + bytes > size)
        return MOE_ERR_INVALID;
    cudaIpcMemHandle_t h;
    if (cudaIpcGetMemHandle(&h, reinterpret_cast<void *>(base)) != cudaSuccess) {
        (void)cudaGetLastError();
        return MOE_ERR_CUDA;
    }
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess)
        return MOE_ERR_CUDA;
    memcpy(out->handle, &h, sizeof(h));
    out->offset = offset;
    out->bytes = bytes;
    out->device = dev;
    return MOE_OK;
}

extern "C" int moe_ipc_open(const moe_ipc_buffer_t *buf, void **ptr, void **mapping)
{
    if (buf == nullptr || ptr == nullptr || mapping == nullptr)
        return MOE_ERR_INVALID;
    cudaIpcMemHandle_t h;
    memcpy(&h, buf->handle, sizeof(h));
    void *base = nullptr;
    if (cudaIpcOpenMemHandle(&base, h, cudaIpcMemLazyEnablePeerAccess) != cudaSuccess) {
        (void)cudaGetLastError();
        return MOE_ERR_CUDA;
    }
    *mapping = base;
    *ptr = static_cast<uint8_t *>(base) + buf->offset;
    return MOE_OK;
}

extern "C" int moe_ipc_close(void *mapping)
{
    if (mapping == nullptr)
        return MOE_ERR_INVALID;
    if (cudaIpcCloseMemHandle(mapping) != cudaSuccess) {
        (void)cudaGetLastError();
        return MOE_ERR_CUDA;
    }
    return MOE_OK;
}
