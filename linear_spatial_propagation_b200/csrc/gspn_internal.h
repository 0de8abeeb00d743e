// gspn_internal.h -- host-side interfaces between the C ABI (gspn_api.cu) and
// the kernel families.  Not part of the public ABI.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/gspn.h"
#include "gspn_common.cuh"

namespace gspn {

constexpr size_t kWsAlign = 256;
inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Validated, normalised view of a descriptor.
struct Problem {
    gspn_desc d;
    Launch g;
    int64_t planes;   // B*C
    int64_t HW;
    size_t elt;       // bytes per element
};

// Device properties the dispatch needs (queried once per device).
struct DeviceInfo {
    int sm_count;
    int max_smem_optin;   // bytes of dynamic shared memory a block may opt in to
};
cudaError_t device_info(DeviceInfo* out);

// Sets the max-dynamic-smem attribute of `fn` once per device.
cudaError_t ensure_smem_attr(const void* fn, int bytes, int slot);

// cuTensorMapEncodeTiled from the driver, looked up once (thread-safe); null
// when the driver does not provide it.
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn encode_tiled();

// Device-side waits of the TMA-fed kernels, process-wide: the limit of every
// wait on data, a stage or a peer warp (gspn_set_wait_limit_ns), and the test
// hook of gspn_set_stall_test (one wait per call on a barrier that nothing
// completes).  Waits that drain copies or release tensor memory keep fixed
// bounds of their own.
struct WaitCfg {
    uint64_t limit_ns;
    int stall;
};
WaitCfg wait_cfg();

// ---- generic kernels (any shape, dtype, mode) ---------------------------------
size_t generic_fwd_workspace(const Problem& p, const DeviceInfo& dev);
gspn_status generic_fwd(const Problem& p, const DeviceInfo& dev, const void* x, const void* logits,
                        const void* lam, void* out, void* ws, cudaStream_t s);
size_t generic_bwd_workspace(const Problem& p, const DeviceInfo& dev);
int generic_bwd_launches(const Problem& p);
gspn_status generic_bwd(const Problem& p, const DeviceInfo& dev, const void* x, const void* logits,
                        const void* lam, const void* dout, void* dx, void* dlogits, void* dlam, void* ws,
                        cudaStream_t s);

// ---- planes of at most 64x64, any mode: one CTA per plane, one warp per direction ----
bool small_eligible(const Problem& p, int backward);
size_t small_bwd_workspace(const Problem& p);
int small_bwd_launches(const Problem& p);
gspn_status small_fwd(const Problem& p, const DeviceInfo& dev, const void* x, const void* logits, const void* lam,
                      void* out, cudaStream_t s);
gspn_status small_bwd(const Problem& p, const DeviceInfo& dev, const void* x, const void* logits, const void* lam,
                      const void* dout, void* dx, void* dlogits, void* dlam, void* ws, cudaStream_t s);

// ---- planes with lines of 65..512 positions: one CTA streams a plane line by line (forward) ----
bool large_eligible(const Problem& p);
size_t large_fwd_workspace(const Problem& p);
gspn_status large_fwd(const Problem& p, const void* x, const void* logits, const void* lam, void* out, void* ws,
                      cudaStream_t s);

// ---- compact 64x64 bf16 forward (TMA-fed, packed fp32x2) ------------------------
bool c64_eligible(const Problem& p);
size_t c64_fwd_workspace(const Problem& p);
gspn_status c64_fwd(const Problem& p, const DeviceInfo& dev, const void* x, const void* logits, const void* lam,
                    void* out, void* ws, cudaStream_t s);
// the same forward on the library's fixed device scratch (no workspace argument)
gspn_status c64_fwd_noalloc(const Problem& p, const DeviceInfo& dev, const void* x, const void* logits,
                            const void* lam, void* out, cudaStream_t s);
// synchronises `s`, then reads the error word of the fixed scratch
gspn_status c64_noalloc_status(cudaStream_t s);

// ---- compact 128x128 bf16 forward (TMA-fed, first arrivals in TMEM) ------------------
bool c128_eligible(const Problem& p);
size_t c128_fwd_workspace(const Problem& p, const DeviceInfo& dev);
gspn_status c128_fwd(const Problem& p, const DeviceInfo& dev, const void* x, const void* logits, const void* lam,
                     void* out, void* ws, cudaStream_t s);

// ---- compact 128x128 bf16 backward (TMA-fed; h_A states in TMEM, a_B through L2) ------
bool c128_bwd_eligible(const Problem& p);
size_t c128_bwd_workspace(const Problem& p, const DeviceInfo& dev);
gspn_status c128_bwd(const Problem& p, const DeviceInfo& dev, const void* x, const void* logits, const void* lam,
                     const void* dout, void* dx, void* dlogits, void* dlam, void* ws, cudaStream_t s);

// ---- compact 64x64 bf16 backward (TMA-fed, checkpointed sweeps) ------------------
bool c64_bwd_eligible(const Problem& p);
size_t c64_bwd_workspace(const Problem& p, const DeviceInfo& dev);
gspn_status c64_bwd(const Problem& p, const DeviceInfo& dev, const void* x, const void* logits, const void* lam,
                    const void* dout, void* dx, void* dlogits, void* dlam, void* ws, cudaStream_t s);

// ---- compressed propagation block (proxy projection, scan, merger, norm, back-projection) ----
size_t block_workspace(const gspn_block_desc* d);
gspn_status block_fwd(const gspn_block_desc* d, const void* x, const void* v, const void* logits, const void* lam,
                      const float* alpha, const float* gamma, const void* u, void* y, void* ws, size_t ws_bytes,
                      cudaStream_t s);

}  // namespace gspn
