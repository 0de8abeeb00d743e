// gspn_large_compact.h -- host-side interface of the compact large-plane
// forward and backward (gspn_large_compact.cu) for the C ABI.  Not part of the public ABI.
#pragma once

#include "gspn_internal.h"

namespace gspn {

// compact bf16 planes with lines of 129..256 positions: one warp per plane
bool lc_eligible(const Problem& p);
size_t lc_fwd_workspace(const Problem& p);
gspn_status lc_fwd(const Problem& p, const DeviceInfo& dev, const void* x, const void* logits, const void* lam,
                   void* out, void* ws, cudaStream_t s);
// the backward of the same planes: states pass, adjoint pass, dlogits (4 launches)
size_t lc_bwd_workspace(const Problem& p);
gspn_status lc_bwd(const Problem& p, const DeviceInfo& dev, const void* x, const void* logits, const void* lam,
                   const void* dout, void* dx, void* dlogits, void* dlam, void* ws, cudaStream_t s);

}  // namespace gspn
