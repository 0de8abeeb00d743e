// gspn_large.cu -- GSPN forward for planes whose lines are longer than the
// on-chip kernels hold (lines of 65 to 512 positions: 256x256 and 512x512
// images at patch 1, or the 16K-scale latents that "Parallel Sequence
// Modeling via Generalized Spatial Propagation Network" targets), any dtype,
// direction set, local-group count and weight mode.
//
// One CTA streams one (b, c) plane line by line.  The line is spread over the
// CTA: lane t of warp w holds positions 2(32w + t) and 2(32w + t) + 1 in
// registers, the neighbours across lanes come from shuffles and those across
// warps from a two-slot edge buffer in shared memory with one CTA barrier per
// line.  Inputs arrive a chunk of lines at a time (8 for bf16, 4 for fp32),
// loaded one chunk ahead:
// * row scans (top->bottom, bottom->top): each line is a row and a lane's two
//   positions are adjacent elements, so a warp reads contiguous bytes;
// * column scans (left->right, right->left): a lane's two positions are two
//   rows, and the chunk's lines are adjacent columns, so each row contributes
//   one 16-byte piece per tensor per chunk.
// The directions of the plane run one after another and merge through an
// fp32 accumulator plane in the workspace (first direction stores, the next
// ones add, the last one adds and writes the output in the I/O dtype), so the
// sum is taken in direction order and does not depend on timing.  Tap weights
// are normalised from the logits (Key design 1) for a whole chunk before its
// lines are walked, so the line loop carries only the dependent update.  With
// channel-shared taps they are formed once per (direction, image, pixel) by a
// pre-kernel, in scan order, and every channel's CTA loads them with its
// chunk instead of recomputing three sigmoids per position and line.
#include "gspn_internal.h"

namespace gspn {

namespace {

constexpr unsigned FULLM = 0xffffffffu;
constexpr int kLargeMaxWarps = 8;  // lines of up to 512 positions

struct LargeArgs {
    Launch g;
    const void* x;
    const void* logits;
    const void* lam;
    void* out;
    float* acc;          // [planes][HW]
    const float2* taps;  // channel-shared taps: [slot][B][line][position] (w0, w2); else unused
    int nw;              // warps per CTA = ceil(max line length / 64)
};

__device__ __forceinline__ float lg_sigmoid(float z) { return __fdividef(1.f, 1.f + __expf(-z)); }

// Channel-shared taps in scan order: taps[((slot*B + b)*L + i)*N + j] = (w0, w2)
// of position j of line i of the slot's direction in image b: the sigmoids of
// the pixel's three tap logits normalised over the taps that exist (w0 = 0 at
// j = 0, w2 = 0 at j = N-1), with the same operations as the in-kernel path.
template <typename T>
__global__ void __launch_bounds__(256) large_taps_kernel(const T* __restrict__ logits, float2* __restrict__ taps,
                                                          const Launch g) {
    const int H = g.H, W = g.W, HW = H * W, B = g.B;
    const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= (int64_t)g.D * B * HW) return;
    const int slot = (int)(idx / ((int64_t)B * HW));
    const int b = (int)(idx / HW % B);
    const int r = (int)(idx % HW);
    const int d = dir_of(g, slot);
    const int N = line_len(d, H, W);
    const int i = r / N, j = r % N;
    const Walk wk = walk_of(d, H, W);
    const int pix = wk.o + i * wk.si + j * wk.sj;
    const T* const lg = logits + ((int64_t)slot * B + b) * 3 * HW;
    const float s0 = j > 0 ? lg_sigmoid(load_elt(lg, pix)) : 0.f;
    const float s1 = lg_sigmoid(load_elt(lg, HW + pix));
    const float s2 = j < N - 1 ? lg_sigmoid(load_elt(lg, 2 * HW + pix)) : 0.f;
    const float rs = __fdividef(1.f, s0 + s1 + s2);
    taps[idx] = make_float2(s0 * rs, s2 * rs);
}

// element access for both dtypes: a chunk is CH elements of one tensor, kept
// as raw 32-bit words (two bf16 or one fp32 per word)
template <typename T>
struct Elt;
template <>
struct Elt<float> {
    static constexpr int CH = 4;  // lines per chunk
    __device__ static float get(const uint32_t* w, int e) { return __uint_as_float(w[e]); }
};
template <>
struct Elt<__nv_bfloat16> {
    static constexpr int CH = 8;
    __device__ static float get(const uint32_t* w, int e) {
        const uint32_t v = w[e >> 1];
        return __uint_as_float((e & 1) ? (v & 0xffff0000u) : (v << 16));
    }
};

// The inputs of one chunk for this lane's two positions: for each of the five
// tensors (x, lambda, logit taps 0..2; with a taps table only x and lambda)
// and each position p, CH values (one per line) packed in WPP words.
template <typename T, bool TAB>
struct Chunk {
    static constexpr int CH = Elt<T>::CH;
    static constexpr int WPP = CH * (int)sizeof(T) / 4;  // words per position and tensor
    static constexpr int NT = TAB ? 2 : 5;
    uint32_t v[NT][2][WPP];
    float4 tw[TAB ? CH : 1];  // with a taps table: (w0, w2) of positions j0, j0 + 1 per line
    float acc[2][CH];  // the accumulator at the chunk's pixels (not the first direction)
};

// The chunk of lines i0 .. i0 + CH - 1 at positions j0, j0 + 1, and, when
// `with_acc`, the accumulator values there.  The accumulator was written by
// this CTA's previous direction, so it is read through the coherent path.
template <typename T, bool TAB>
__device__ __forceinline__ void load_chunk(Chunk<T, TAB>& ck, const T* const (&src)[5], const float2* tap,
                                           const float* acc, bool with_acc, bool rowscan, const Walk& wk, int W,
                                           int i0, int j0, int N) {
    constexpr int CH = Elt<T>::CH;
    constexpr int WPP = Chunk<T, TAB>::WPP;
    constexpr int NT = Chunk<T, TAB>::NT;
    if constexpr (TAB) {
        // the taps of lines i0 .. i0 + CH - 1 at positions j0, j0 + 1: 16 bytes per line
#pragma unroll
        for (int e = 0; e < CH; ++e)
            ck.tw[e] = j0 < N ? __ldg(reinterpret_cast<const float4*>(tap + (size_t)(i0 + e) * N + j0))
                              : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    if (rowscan) {
        // line i0 + e: a row; positions j0, j0 + 1 are adjacent elements
#pragma unroll
        for (int e = 0; e < CH; ++e) {
            const int pix = wk.o + (i0 + e) * wk.si + j0;
            float2 av = make_float2(0.f, 0.f);
            if (with_acc && j0 < N) av = *reinterpret_cast<const float2*>(acc + pix);  // j0 + 1 < N too: N is even
            ck.acc[0][e] = av.x;
            ck.acc[1][e] = av.y;
#pragma unroll
            for (int s = 0; s < NT; ++s) {
                const uint16_t* b16 = reinterpret_cast<const uint16_t*>(src[s] + pix);
                if constexpr (sizeof(T) == 4) {
                    const float* f = reinterpret_cast<const float*>(src[s]) + pix;
                    ck.v[s][0][e] = __float_as_uint(j0 < N ? __ldg(f) : 0.f);
                    ck.v[s][1][e] = __float_as_uint(j0 + 1 < N ? __ldg(f + 1) : 0.f);
                } else {
                    const uint32_t lo = j0 < N ? (uint32_t)__ldg(b16) : 0u;
                    const uint32_t hi = j0 + 1 < N ? (uint32_t)__ldg(b16 + 1) : 0u;
                    // value e of position p sits in half (e & 1) of word e >> 1
                    if (e & 1) {
                        ck.v[s][0][e >> 1] |= lo << 16;
                        ck.v[s][1][e >> 1] |= hi << 16;
                    } else {
                        ck.v[s][0][e >> 1] = lo;
                        ck.v[s][1][e >> 1] = hi;
                    }
                }
            }
        }
    } else {
        // lines i0 .. i0 + CH - 1: CH adjacent columns of the rows j0, j0 + 1;
        // left->right (si = +1) reads them ascending, right->left (si = -1)
        // descending, so the piece starts at the chunk's lowest column
#pragma unroll
        for (int p = 0; p < 2; ++p) {
            const int j = j0 + p;
            const int first = wk.si > 0 ? wk.o + i0 + j * wk.sj : wk.o - (i0 + CH - 1) + j * wk.sj;
            // the accumulator of these CTA pixels, in line order
            float av[CH];
#pragma unroll
            for (int m = 0; m < CH; m += 4) {
                float4 q = make_float4(0.f, 0.f, 0.f, 0.f);
                if (with_acc && j < N) q = *reinterpret_cast<const float4*>(acc + first + m);
                av[m] = q.x;
                av[m + 1] = q.y;
                av[m + 2] = q.z;
                av[m + 3] = q.w;
            }
            if (wk.si > 0) {
#pragma unroll
                for (int m = 0; m < CH; ++m) ck.acc[p][m] = av[m];
            } else {
#pragma unroll
                for (int m = 0; m < CH; ++m) ck.acc[p][m] = av[CH - 1 - m];
            }
#pragma unroll
            for (int s = 0; s < NT; ++s) {
                uint4 q = make_uint4(0u, 0u, 0u, 0u);
                if (j < N) q = __ldg(reinterpret_cast<const uint4*>(src[s] + first));
                uint32_t w[4] = {q.x, q.y, q.z, q.w};
                if (wk.si > 0) {
#pragma unroll
                    for (int u = 0; u < WPP; ++u) ck.v[s][p][u] = w[u];
                } else {
                    // reverse the element order of the piece
#pragma unroll
                    for (int u = 0; u < WPP; ++u) {
                        const uint32_t r = w[WPP - 1 - u];
                        ck.v[s][p][u] = sizeof(T) == 4 ? r : __byte_perm(r, 0, 0x1032);
                    }
                }
            }
        }
    }
}

template <typename T, bool TAB>
__global__ void __launch_bounds__(kLargeMaxWarps * 32) large_fwd_kernel(const LargeArgs a) {
    constexpr int CH = Elt<T>::CH;
    constexpr int NTAP0 = TAB ? 0 : 2;  // first logit tensor of a chunk (the in-kernel taps)
    __shared__ float edge[2][kLargeMaxWarps][2];  // [line parity][warp][first, last]
    const int warp = threadIdx.x >> 5, t = threadIdx.x & 31;
    const int H = a.g.H, W = a.g.W, HW = H * W, B = a.g.B, C = a.g.C;
    const int64_t plane = blockIdx.x;
    const int64_t b = plane / C, c = plane % C, cw = a.g.shared ? 0 : c;
    const int Cw = a.g.shared ? 1 : C;
    const int j0 = 2 * (32 * warp + t);
    float* const acc = a.acc + plane * HW;
    T* const out = static_cast<T*>(a.out) + plane * HW;

    for (int slot = 0; slot < a.g.D; ++slot) {
        const int d = dir_of(a.g, slot);
        const bool rowscan = d < 2;
        const int L = scan_len(d, H, W), N = line_len(d, H, W), seg = L / a.g.groups;
        const Walk wk = walk_of(d, H, W);
        const T* const lg = static_cast<const T*>(a.logits) + ((slot * (int64_t)B + b) * Cw + cw) * 3 * HW;
        const T* const src[5] = {static_cast<const T*>(a.x) + plane * HW,
                                 static_cast<const T*>(a.lam) + ((slot * (int64_t)B + b) * C + c) * HW, lg,
                                 lg + HW, lg + 2 * HW};
        const float2* const tap = TAB ? a.taps + (slot * (int64_t)B + b) * HW : nullptr;
        const bool first_dir = slot == 0, last_dir = slot == a.g.D - 1;
        float h0 = 0.f, h1 = 0.f;
        int gpos = 0;
        Chunk<T, TAB> cur, nxt;
        load_chunk<T, TAB>(cur, src, tap, acc, !first_dir, rowscan, wk, W, 0, j0, N);
        float colbuf[2][CH];  // column scans: a chunk of outputs per row, stored at the chunk's end
        for (int i0 = 0; i0 < L; i0 += CH) {
            if (i0 + CH < L) load_chunk<T, TAB>(nxt, src, tap, acc, !first_dir, rowscan, wk, W, i0 + CH, j0, N);
            // the chunk's taps and lambda * x first: they do not depend on the
            // state, so the sigmoids of all its lines and positions overlap, and
            // the line loop below is only the dependent update
            float w0c[CH][2], w2c[CH][2], uc[CH][2];
#pragma unroll
            for (int e = 0; e < CH; ++e)
#pragma unroll
                for (int p = 0; p < 2; ++p) {
                    const int j = j0 + p;
                    uc[e][p] = Elt<T>::get(cur.v[1][p], e) * Elt<T>::get(cur.v[0][p], e);
                    if constexpr (TAB) {
                        w0c[e][p] = p ? cur.tw[e].z : cur.tw[e].x;
                        w2c[e][p] = p ? cur.tw[e].w : cur.tw[e].y;
                    } else {
                        const float s0 = j > 0 ? lg_sigmoid(Elt<T>::get(cur.v[NTAP0][p], e)) : 0.f;
                        const float s1 = lg_sigmoid(Elt<T>::get(cur.v[NTAP0 + 1][p], e));
                        const float s2 = j < N - 1 ? lg_sigmoid(Elt<T>::get(cur.v[NTAP0 + 2][p], e)) : 0.f;
                        const float r = __fdividef(1.f, s0 + s1 + s2);
                        w0c[e][p] = s0 * r;
                        w2c[e][p] = s2 * r;
                    }
                }
#pragma unroll
            for (int e = 0; e < CH; ++e) {
                const int i = i0 + e;
                const int par = i & 1;
                // neighbours of the previous line: lanes by shuffles, warps by the edge buffer
                float hl = __shfl_up_sync(FULLM, h1, 1);
                float hr = __shfl_down_sync(FULLM, h0, 1);
                if (a.nw > 1) {
                    if (t == 0) hl = warp > 0 ? edge[par ^ 1][warp - 1][1] : 0.f;
                    if (t == 31) hr = warp + 1 < a.nw ? edge[par ^ 1][warp + 1][0] : 0.f;
                }
                // h' = u + w0 h[j-1] + (1 - w0 - w2) h[j] + w2 h[j+1]; h_{-1} = 0 at a
                // scan or group start; positions beyond the line stay 0
                float hn[2];
                if (gpos == 0) {
                    hn[0] = uc[e][0];
                    hn[1] = uc[e][1];
                } else {
                    hn[0] = uc[e][0] + h0 + w0c[e][0] * (hl - h0) + w2c[e][0] * (h1 - h0);
                    hn[1] = uc[e][1] + h1 + w0c[e][1] * (h0 - h1) + w2c[e][1] * (hr - h1);
                }
                h0 = j0 < N ? hn[0] : 0.f;
                h1 = j0 + 1 < N ? hn[1] : 0.f;
                hn[0] = h0;
                hn[1] = h1;
                if (a.nw > 1) {
                    if (t == 0) edge[par][warp][0] = h0;
                    if (t == 31) edge[par][warp][1] = h1;
                    __syncthreads();
                }
                gpos = gpos + 1 == seg ? 0 : gpos + 1;
                if (rowscan) {
                    // this line's two values: adjacent elements of one row
                    const int pix = wk.o + i * wk.si + j0;
#pragma unroll
                    for (int p = 0; p < 2; ++p) {
                        if (j0 + p >= N) continue;
                        const float v = hn[p] + cur.acc[p][e];  // 0 for the first direction
                        if (last_dir)
                            store_elt(out, pix + p, v);
                        else
                            acc[pix + p] = v;
                    }
                } else {
                    colbuf[0][e] = h0 + cur.acc[0][e];
                    colbuf[1][e] = h1 + cur.acc[1][e];
                }
            }
            if (!rowscan) {
                // the chunk's CH lines are CH adjacent columns of rows j0, j0 + 1
#pragma unroll
                for (int p = 0; p < 2; ++p) {
                    const int j = j0 + p;
                    if (j >= N) continue;
                    const int first = wk.si > 0 ? wk.o + i0 + j * wk.sj : wk.o - (i0 + CH - 1) + j * wk.sj;
                    float v[CH];
                    if (wk.si > 0) {
#pragma unroll
                        for (int m = 0; m < CH; ++m) v[m] = colbuf[p][m];
                    } else {
#pragma unroll
                        for (int m = 0; m < CH; ++m) v[m] = colbuf[p][CH - 1 - m];
                    }
                    if (last_dir) {
#pragma unroll
                        for (int m = 0; m < CH; ++m) store_elt(out, first + m, v[m]);
                    } else {
#pragma unroll
                        for (int m = 0; m < CH; m += 4)
                            *reinterpret_cast<float4*>(acc + first + m) = make_float4(v[m], v[m + 1], v[m + 2], v[m + 3]);
                    }
                }
            }
            cur = nxt;
        }
        // every line of this direction is in acc before the next direction reads it
        __syncthreads();
    }
}

}  // namespace

// Lines of 65..512 positions whose planes do not fit the on-chip kernels;
// H and W multiples of 8 so that a chunk's pieces of a row are whole 16-byte
// loads.
bool large_eligible(const Problem& p) {
    const int H = p.g.H, W = p.g.W;
    const int nmax = H > W ? H : W;
    return nmax > 64 && nmax <= 64 * kLargeMaxWarps && H % 8 == 0 && W % 8 == 0 && p.HW <= (1 << 24);
}

// the accumulator planes, then (channel-shared taps) the taps table
size_t large_fwd_workspace(const Problem& p) {
    const size_t acc = align_up((size_t)p.planes * p.HW * sizeof(float), kWsAlign);
    return acc + (p.g.shared ? align_up((size_t)p.g.D * p.g.B * p.HW * sizeof(float2), kWsAlign) : 0);
}

gspn_status large_fwd(const Problem& p, const void* x, const void* logits, const void* lam, void* out, void* ws,
                      cudaStream_t s) {
    LargeArgs a;
    a.g = p.g;
    a.x = x;
    a.logits = logits;
    a.lam = lam;
    a.out = out;
    a.acc = static_cast<float*>(ws);
    a.taps = nullptr;
    const int nmax = p.g.H > p.g.W ? p.g.H : p.g.W;
    a.nw = (nmax + 63) / 64;
    if (p.planes > 0x7fffffff) return GSPN_ERR_UNSUPPORTED;
    const unsigned grid = (unsigned)p.planes;
    const bool f32 = p.d.dtype == GSPN_F32;
    if (p.g.shared) {
        float2* taps = reinterpret_cast<float2*>(static_cast<char*>(ws) +
                                                 align_up((size_t)p.planes * p.HW * sizeof(float), kWsAlign));
        const int64_t n = (int64_t)p.g.D * p.g.B * p.HW;
        const unsigned tg = (unsigned)((n + 255) / 256);
        if (f32)
            large_taps_kernel<float><<<tg, 256, 0, s>>>(static_cast<const float*>(logits), taps, p.g);
        else
            large_taps_kernel<__nv_bfloat16><<<tg, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(logits), taps, p.g);
        if (cudaGetLastError() != cudaSuccess) return GSPN_ERR_CUDA;
        a.taps = taps;
        if (f32)
            large_fwd_kernel<float, true><<<grid, a.nw * 32, 0, s>>>(a);
        else
            large_fwd_kernel<__nv_bfloat16, true><<<grid, a.nw * 32, 0, s>>>(a);
    } else {
        if (f32)
            large_fwd_kernel<float, false><<<grid, a.nw * 32, 0, s>>>(a);
        else
            large_fwd_kernel<__nv_bfloat16, false><<<grid, a.nw * 32, 0, s>>>(a);
    }
    return cudaGetLastError() == cudaSuccess ? GSPN_OK : GSPN_ERR_CUDA;
}

}  // namespace gspn
