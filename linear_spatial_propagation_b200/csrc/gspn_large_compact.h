// gspn_large_compact.h -- host-side interface of the compact large-plane
// forward (gspn_large_compact.cu) for the C ABI.  Not part of the public ABI.
#pragma once

#include "gspn_internal.h"

namespace gspn {

// compact bf16 planes with lines of 129..256 positions: one warp per plane (forward)
bool lc_eligible(const Problem& p);
size_t lc_fwd_workspace(const Problem& p);
gspn_status lc_fwd(const Problem& p, const DeviceInfo& dev, const void* x, const void* logits, const void* lam,
                   void* out, void* ws, cudaStream_t s);

}  // namespace gspn
