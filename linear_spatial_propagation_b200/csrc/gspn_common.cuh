// gspn_common.cuh -- device helpers shared by the libgspn kernels.
//
// Coordinates (GSPN, "Parallel Sequence Modeling via Generalized Spatial
// Propagation Network", Key design 2: row and column line scans in four
// directions).  For direction d, line i in scan order and position j along the
// line, the image pixel (r, c) is
//     T2B (i, j) -> (i, j)        B2T (i, j) -> (H-1-i, j)
//     L2R (i, j) -> (j, i)        R2L (i, j) -> (j, W-1-i)
// and tap k in {0,1,2} of position j reads position j+k-1 of line i-1.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace gspn {

enum Dir { T2B = 0, B2T = 1, L2R = 2, R2L = 3 };

__host__ __device__ __forceinline__ int scan_len(int d, int H, int W) { return d < 2 ? H : W; }
__host__ __device__ __forceinline__ int line_len(int d, int H, int W) { return d < 2 ? W : H; }

// offset r*W + c of scan coordinate (i, j) in direction d
__host__ __device__ __forceinline__ int pix(int d, int H, int W, int i, int j) {
    switch (d) {
    case T2B: return i * W + j;
    case B2T: return (H - 1 - i) * W + j;
    case L2R: return j * W + i;
    default: return j * W + (W - 1 - i);
    }
}

// The same map as an offset o + i*si + j*sj, for loops that walk a direction
// without a branch per access.
struct Walk {
    int o, si, sj;
};
__host__ __device__ __forceinline__ Walk walk_of(int d, int H, int W) {
    return d == T2B ? Walk{0, W, 1} : d == B2T ? Walk{(H - 1) * W, -W, 1} : d == L2R ? Walk{0, 1, W} : Walk{W - 1, -1, W};
}

// ---- element access ---------------------------------------------------------
// bf16 <-> fp32: a bf16 value is the top 16 bits of the fp32 with the same value.
__device__ __forceinline__ float bf16_bits_to_float(uint16_t u) { return __uint_as_float(((uint32_t)u) << 16); }

__device__ __forceinline__ float load_elt(const float* p, int64_t i) { return __ldg(p + i); }
__device__ __forceinline__ float load_elt(const __nv_bfloat16* p, int64_t i) {
    return bf16_bits_to_float(__ldg(reinterpret_cast<const unsigned short*>(p) + i));
}
__device__ __forceinline__ void store_elt(float* p, int64_t i, float v) { p[i] = v; }
__device__ __forceinline__ void store_elt(__nv_bfloat16* p, int64_t i, float v) { p[i] = __float2bfloat16_rn(v); }

// ---- gate ---------------------------------------------------------------------
// Sigmoid of a tap logit (GSPN Key design 1: "sigmoid on the non-zero entries
// of each row, then row normalisation").  __expf's error is a few ulp; the
// result is exact 0 for logits below about -88.
__device__ __forceinline__ float sigmoidf(float z) { return 1.0f / (1.0f + __expf(-z)); }

// ---- deterministic channel sums --------------------------------------------
// Tap gradients summed over channels (channel-shared taps) accumulate as 64-bit
// fixed-point integers with a resolution of 2^-32: integer addition is
// associative, so the sums do not depend on the order in which planes arrive.
// A value v adds round(v * 2^32); |v| and every partial sum must stay below
// 2^31.  The quantisation (2^-33 per term at most) is far below fp32 rounding
// for values above 2^-8.
__device__ __forceinline__ void fix_add(unsigned long long* p, float v) {
    atomicAdd(p, (unsigned long long)__float2ll_rn(v * 4294967296.0f));
}
__device__ __forceinline__ float fix_value(unsigned long long s) {
    return (float)((double)(long long)s * (1.0 / 4294967296.0));
}

struct Launch {
    int B, C, H, W;
    int D;            // number of enabled directions
    int dirs[4];      // direction of each D slot, in bit order
    int groups;
    int shared;       // 1: logits have one channel (Cw = 1)
};

// Direction of slot `slot` < 4.  A chain of selects, not an index: indexing the
// array with a runtime value would copy the kernel's parameter block into
// local memory.
__device__ __forceinline__ int dir_of(const Launch& g, int slot) {
    return slot == 0 ? g.dirs[0] : slot == 1 ? g.dirs[1] : slot == 2 ? g.dirs[2] : g.dirs[3];
}

}  // namespace gspn
