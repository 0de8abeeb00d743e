// gspn_api.cu -- the C ABI of libgspn (declared in include/gspn.h): argument
// checks, workspace sizing and dispatch to a kernel family.  Every check runs
// on the host before any launch; no exception crosses the ABI.
#include <atomic>
#include <cstdint>
#include <cstring>

#include "gspn_internal.h"
#include "gspn_large_compact.h"

namespace gspn {

namespace {

constexpr int kMaxDevices = 64;
constexpr uint64_t kDefaultWaitLimitNs = 2000000000ull;  // 2 s
constexpr int kMaxAttrSlots = 48;

struct DevCache {
    std::atomic<int> ready{0};
    DeviceInfo info{};
};
DevCache g_dev[kMaxDevices];
std::atomic<int> g_attr[kMaxDevices][kMaxAttrSlots];

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

gspn_status validate(const gspn_desc* d, Problem* p) {
    if (!d) return GSPN_ERR_INVALID_ARG;
    if (d->B < 1 || d->C < 1 || d->H < 1 || d->W < 1) return GSPN_ERR_INVALID_ARG;
    if ((d->dir_mask & 15u) == 0 || (d->dir_mask & ~15u)) return GSPN_ERR_INVALID_ARG;
    if (d->groups < 1) return GSPN_ERR_INVALID_ARG;
    if ((d->dir_mask & 3u) && d->H % d->groups) return GSPN_ERR_INVALID_ARG;
    if ((d->dir_mask & 12u) && d->W % d->groups) return GSPN_ERR_INVALID_ARG;
    if (d->dtype != GSPN_F32 && d->dtype != GSPN_BF16) return GSPN_ERR_UNSUPPORTED;
    // the kernels index a plane with 32-bit ints and tensors with 64-bit ones
    if (d->H > (1 << 20) || d->W > (1 << 20) || d->H * d->W > (int64_t)1 << 30) return GSPN_ERR_INVALID_ARG;
    if (d->B > (1 << 30) || d->C > (1 << 30)) return GSPN_ERR_INVALID_ARG;
    const int D = __builtin_popcount(d->dir_mask & 15u);
    const int64_t HW = d->H * d->W;
    if (d->B * d->C > ((int64_t)1 << 40) / HW / (D * 3)) return GSPN_ERR_INVALID_ARG;
    if (p) {
        std::memset(p, 0, sizeof(*p));
        p->d = *d;
        p->g.B = (int)d->B;
        p->g.C = (int)d->C;
        p->g.H = (int)d->H;
        p->g.W = (int)d->W;
        p->g.D = D;
        int s = 0;
        for (int k = 0; k < 4; ++k)
            if (d->dir_mask & (1u << k)) p->g.dirs[s++] = k;
        p->g.groups = d->groups;
        p->g.shared = d->shared_weights ? 1 : 0;
        p->planes = d->B * d->C;
        p->HW = HW;
        p->elt = d->dtype == GSPN_F32 ? 4 : 2;
    }
    return GSPN_OK;
}

gspn_status check_ptrs(std::initializer_list<const void*> ptrs) {
    for (const void* q : ptrs)
        if (!q) return GSPN_ERR_INVALID_ARG;
    for (const void* q : ptrs)
        if (!aligned16(q)) return GSPN_ERR_ALIGNMENT;
    return GSPN_OK;
}

gspn_status check_ws(void* ws, size_t have, size_t need) {
    if (need == 0) return GSPN_OK;
    if (!ws || have < need) return GSPN_ERR_WORKSPACE;
    if (reinterpret_cast<uintptr_t>(ws) % kWsAlign) return GSPN_ERR_ALIGNMENT;
    return GSPN_OK;
}

// The kernel family a descriptor runs on: the TMA-fed compact kernels for their
// shapes (64x64, 128x128, and compact planes with lines of 129..256), the
// one-CTA-per-plane kernels for planes of at most 64x64, the large-plane
// forward for the other lines of 65..512, the generic kernels for everything
// else.
enum class Path { kC64, kC128, kSmall, kLargeCompact, kLarge, kGeneric };
Path pick(const Problem& p, int backward) {
    if (backward ? c64_bwd_eligible(p) : c64_eligible(p)) return Path::kC64;
    if (backward ? c128_bwd_eligible(p) : c128_eligible(p)) return Path::kC128;
    if (small_eligible(p, backward)) return Path::kSmall;
    if (lc_eligible(p)) return Path::kLargeCompact;
    if (!backward && large_eligible(p)) return Path::kLarge;
    return Path::kGeneric;
}

std::atomic<uint64_t> g_wait_limit_ns{kDefaultWaitLimitNs};
std::atomic<int> g_stall_test{0};
std::atomic<int> g_sync_check{0};

// The error word a TMA-fed kernel family sets when a bounded wait expires sits
// at offset 0 of its workspace; the other families have no device-side waits.
bool has_status_word(Path path) {
    return path == Path::kC64 || path == Path::kC128 || path == Path::kLargeCompact;
}

// Synchronises `s` and maps the call's outcome to a status: a CUDA error, an
// expired wait recorded in the error word at `word` (null: none), or OK.
gspn_status sync_status(const void* word, cudaStream_t s) {
    int v = 0;
    if (word && cudaMemcpyAsync(&v, word, sizeof(v), cudaMemcpyDeviceToHost, s) != cudaSuccess) return GSPN_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return GSPN_ERR_CUDA;
    return v ? GSPN_ERR_TIMEOUT : GSPN_OK;
}

}  // namespace

EncodeTiledFn encode_tiled() {
    // a function-local static: initialised exactly once, even under concurrent first calls
    static const EncodeTiledFn fn = []() -> EncodeTiledFn {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return nullptr;
        return reinterpret_cast<EncodeTiledFn>(p);
    }();
    return fn;
}

WaitCfg wait_cfg() {
    return WaitCfg{g_wait_limit_ns.load(std::memory_order_relaxed), g_stall_test.load(std::memory_order_relaxed)};
}

cudaError_t device_info(DeviceInfo* out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    DevCache& c = g_dev[dev];
    if (!c.ready.load(std::memory_order_acquire)) {
        DeviceInfo info;
        e = cudaDeviceGetAttribute(&info.sm_count, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return e;
        e = cudaDeviceGetAttribute(&info.max_smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
        if (e != cudaSuccess) return e;
        c.info = info;
        c.ready.store(1, std::memory_order_release);
    }
    *out = c.info;
    return cudaSuccess;
}

cudaError_t ensure_smem_attr(const void* fn, int bytes, int slot) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices || slot < 0 || slot >= kMaxAttrSlots) return cudaErrorInvalidValue;
    std::atomic<int>& a = g_attr[dev][slot];
    if (a.load(std::memory_order_acquire) >= bytes) return cudaSuccess;
    // always raise to the device maximum once, so later calls need no attribute change
    DeviceInfo di;
    e = device_info(&di);
    if (e != cudaSuccess) return e;
    const int want = bytes > di.max_smem_optin ? bytes : di.max_smem_optin;
    e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, want);
    if (e != cudaSuccess) return e;
    a.store(want, std::memory_order_release);
    return cudaSuccess;
}

}  // namespace gspn

using namespace gspn;

extern "C" {

int gspn_version(void) { return 100; }

const char* gspn_status_string(gspn_status s) {
    switch (s) {
    case GSPN_OK: return "ok";
    case GSPN_ERR_INVALID_ARG: return "invalid argument";
    case GSPN_ERR_UNSUPPORTED: return "unsupported configuration";
    case GSPN_ERR_ALIGNMENT: return "pointer not aligned (tensors: 16 bytes, workspace: 256 bytes)";
    case GSPN_ERR_WORKSPACE: return "workspace missing or too small";
    case GSPN_ERR_CUDA: return "CUDA runtime error";
    case GSPN_ERR_TIMEOUT: return "device-side wait timed out";
    case GSPN_ERR_SCRATCH_LIMIT:
        return "problem exceeds the fixed scratch of gspn_fwd_noalloc (compact 64x64 bf16 forward, B <= 32)";
    default: return "unknown status";
    }
}

size_t gspn_workspace_size(const gspn_desc* desc, int backward) {
    Problem p;
    if (validate(desc, &p) != GSPN_OK) return 0;
    DeviceInfo dev;
    if (device_info(&dev) != cudaSuccess) return 0;
    switch (pick(p, backward)) {
    case Path::kC64: return backward ? c64_bwd_workspace(p, dev) : c64_fwd_workspace(p);
    case Path::kC128: return backward ? c128_bwd_workspace(p, dev) : c128_fwd_workspace(p, dev);
    case Path::kSmall: return backward ? small_bwd_workspace(p) : 0;
    case Path::kLargeCompact: return backward ? lc_bwd_workspace(p) : lc_fwd_workspace(p);
    case Path::kLarge: return large_fwd_workspace(p);
    default: return backward ? generic_bwd_workspace(p, dev) : generic_fwd_workspace(p, dev);
    }
}

int gspn_launches_per_call(const gspn_desc* desc, int backward) {
    Problem p;
    if (validate(desc, &p) != GSPN_OK) return 0;
    switch (pick(p, backward)) {
    case Path::kC64:
    case Path::kC128: return backward ? 3 : 2;
    case Path::kSmall: return backward ? small_bwd_launches(p) : 1;
    case Path::kLargeCompact: return backward ? 4 : 2;  // the taps table, then the scan (backward: states, adjoint, dlogits)
    case Path::kLarge: return p.g.shared ? 2 : 1;  // channel-shared taps: the taps pre-kernel first
    default: return backward ? generic_bwd_launches(p) : 1;
    }
}

const char* gspn_variant_name(const gspn_desc* desc, int backward) {
    Problem p;
    if (validate(desc, &p) != GSPN_OK) return "invalid";
    switch (pick(p, backward)) {
    case Path::kC64: return backward ? "compact64_tma_bwd" : "compact64_tma_fwd";
    case Path::kC128: return backward ? "compact128_tma_bwd" : "compact128_tma_fwd";
    case Path::kSmall: return backward ? "small_plane_bwd" : "small_plane_fwd";
    case Path::kLargeCompact: return backward ? "large_compact_bwd" : "large_compact_fwd";
    case Path::kLarge: return "large_plane_fwd";
    default: return backward ? "generic_bwd" : "generic_fwd";
    }
}

gspn_status gspn_fwd(const gspn_desc* desc, const void* x, const void* logits, const void* lambda, void* out,
                     void* workspace, size_t ws_bytes, void* stream) {
    Problem p;
    gspn_status st = validate(desc, &p);
    if (st != GSPN_OK) return st;
    st = check_ptrs({x, logits, lambda, out});
    if (st != GSPN_OK) return st;
    DeviceInfo dev;
    if (device_info(&dev) != cudaSuccess) return GSPN_ERR_CUDA;
    const Path path = pick(p, 0);
    st = check_ws(workspace, ws_bytes,
                  path == Path::kC64    ? c64_fwd_workspace(p)
                  : path == Path::kC128 ? c128_fwd_workspace(p, dev)
                  : path == Path::kSmall ? 0
                  : path == Path::kLargeCompact ? lc_fwd_workspace(p)
                  : path == Path::kLarge ? large_fwd_workspace(p)
                                         : generic_fwd_workspace(p, dev));
    if (st != GSPN_OK) return st;
    const cudaStream_t cs = static_cast<cudaStream_t>(stream);
    st = path == Path::kC64    ? c64_fwd(p, dev, x, logits, lambda, out, workspace, cs)
         : path == Path::kC128 ? c128_fwd(p, dev, x, logits, lambda, out, workspace, cs)
         : path == Path::kSmall ? small_fwd(p, dev, x, logits, lambda, out, cs)
         : path == Path::kLargeCompact ? lc_fwd(p, dev, x, logits, lambda, out, workspace, cs)
         : path == Path::kLarge ? large_fwd(p, x, logits, lambda, out, workspace, cs)
                                : generic_fwd(p, dev, x, logits, lambda, out, workspace, cs);
    if (st != GSPN_OK || !g_sync_check.load(std::memory_order_relaxed)) return st;
    return sync_status(has_status_word(path) ? workspace : nullptr, cs);
}

gspn_status gspn_fwd_noalloc(const gspn_desc* desc, const void* x, const void* logits, const void* lambda, void* out,
                             void* stream) {
    Problem p;
    gspn_status st = validate(desc, &p);
    if (st != GSPN_OK) return st;
    st = check_ptrs({x, logits, lambda, out});
    if (st != GSPN_OK) return st;
    DeviceInfo dev;
    if (device_info(&dev) != cudaSuccess) return GSPN_ERR_CUDA;
    const cudaStream_t cs = static_cast<cudaStream_t>(stream);
    st = c64_fwd_noalloc(p, dev, x, logits, lambda, out, cs);
    if (st != GSPN_OK || !g_sync_check.load(std::memory_order_relaxed)) return st;
    return c64_noalloc_status(cs);
}

gspn_status gspn_noalloc_status(void* stream) { return c64_noalloc_status(static_cast<cudaStream_t>(stream)); }

gspn_status gspn_device_status(const gspn_desc* desc, int backward, const void* workspace, void* stream) {
    Problem p;
    gspn_status st = validate(desc, &p);
    if (st != GSPN_OK) return st;
    const bool word = has_status_word(pick(p, backward));
    if (word && !workspace) return GSPN_ERR_INVALID_ARG;
    return sync_status(word ? workspace : nullptr, static_cast<cudaStream_t>(stream));
}

size_t gspn_block_workspace_size(const gspn_block_desc* desc) { return block_workspace(desc); }

gspn_status gspn_block_fwd(const gspn_block_desc* desc, const void* x, const void* v_proj, const void* logits,
                           const void* lambda, const float* alpha, const float* gamma, const void* u_proj, void* y,
                           void* workspace, size_t ws_bytes, void* stream) {
    const cudaStream_t cs = static_cast<cudaStream_t>(stream);
    gspn_status st = block_fwd(desc, x, v_proj, logits, lambda, alpha, gamma, u_proj, y, workspace, ws_bytes, cs);
    if (st != GSPN_OK || !g_sync_check.load(std::memory_order_relaxed)) return st;
    return sync_status(workspace, cs);
}

gspn_status gspn_block_device_status(const gspn_block_desc* desc, const void* workspace, void* stream) {
    if (block_workspace(desc) == 0) return GSPN_ERR_INVALID_ARG;
    if (!workspace) return GSPN_ERR_INVALID_ARG;
    return sync_status(workspace, static_cast<cudaStream_t>(stream));
}

uint64_t gspn_set_wait_limit_ns(uint64_t limit_ns) {
    return g_wait_limit_ns.exchange(limit_ns ? limit_ns : kDefaultWaitLimitNs);
}

int gspn_set_sync_check(int on) { return g_sync_check.exchange(on ? 1 : 0); }

int gspn_set_stall_test(int on) { return g_stall_test.exchange(on ? 1 : 0); }

gspn_status gspn_bwd(const gspn_desc* desc, const void* x, const void* logits, const void* lambda,
                     const void* dout, void* dx, void* dlogits, void* dlambda, void* workspace, size_t ws_bytes,
                     void* stream) {
    Problem p;
    gspn_status st = validate(desc, &p);
    if (st != GSPN_OK) return st;
    st = check_ptrs({x, logits, lambda, dout, dx, dlogits, dlambda});
    if (st != GSPN_OK) return st;
    DeviceInfo dev;
    if (device_info(&dev) != cudaSuccess) return GSPN_ERR_CUDA;
    const Path path = pick(p, 1);
    st = check_ws(workspace, ws_bytes,
                  path == Path::kC64     ? c64_bwd_workspace(p, dev)
                  : path == Path::kC128  ? c128_bwd_workspace(p, dev)
                  : path == Path::kSmall ? small_bwd_workspace(p)
                  : path == Path::kLargeCompact ? lc_bwd_workspace(p)
                                         : generic_bwd_workspace(p, dev));
    if (st != GSPN_OK) return st;
    const cudaStream_t cs = static_cast<cudaStream_t>(stream);
    st = path == Path::kC64     ? c64_bwd(p, dev, x, logits, lambda, dout, dx, dlogits, dlambda, workspace, cs)
         : path == Path::kC128  ? c128_bwd(p, dev, x, logits, lambda, dout, dx, dlogits, dlambda, workspace, cs)
         : path == Path::kSmall ? small_bwd(p, dev, x, logits, lambda, dout, dx, dlogits, dlambda, workspace, cs)
         : path == Path::kLargeCompact ? lc_bwd(p, dev, x, logits, lambda, dout, dx, dlogits, dlambda, workspace, cs)
                                : generic_bwd(p, dev, x, logits, lambda, dout, dx, dlogits, dlambda, workspace, cs);
    if (st != GSPN_OK || !g_sync_check.load(std::memory_order_relaxed)) return st;
    return sync_status(has_status_word(path) ? workspace : nullptr, cs);
}

}  // extern "C"
