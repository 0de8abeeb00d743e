// gspn_internal.h -- host-side interfaces between the C ABI (gspn_api.cu) and
// the kernel families.  Not part of the public ABI.
#pragma once

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

// ---- compact 64x64 bf16 forward (TMA-fed, packed fp32x2) ------------------------
bool c64_eligible(const Problem& p);
size_t c64_fwd_workspace(const Problem& p);
gspn_status c64_fwd(const Problem& p, const DeviceInfo& dev, const void* x, const void* logits, const void* lam,
                    void* out, void* ws, cudaStream_t s);
// the same forward on the library's fixed device scratch (no workspace argument)
gspn_status c64_fwd_noalloc(const Problem& p, const DeviceInfo& dev, const void* x, const void* logits,
                            const void* lam, void* out, cudaStream_t s);

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

}  // namespace gspn
