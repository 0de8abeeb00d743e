// gspn_block.cu -- the compressed propagation block around the GSPN scan.
//
// What it computes ("GSPN-2: Efficient Parallel Sequence Modeling", OpenReview
// response, "Relate Compressive Proxy Dimension to Low-rank Approximation":
// x in R^{N x C x H x W} goes through a lightweight linear layer to C_proxy
// channels, the recurrence runs there, and the result is projected back to C;
// "Parallel Sequence Modeling via Generalized Spatial Propagation Network",
// Key design 2: the four directions are aggregated by a learnable merger;
// "Scaling Parallel Sequence Models to Vision Foundation Models", abstract: a
// compressed latent-space propagation block with fused normalisation):
//
//   xp[b,k]  = sum_c V[k,c] x[b,c]                         (proxy projection)
//   h_d[b,k] = GSPN scan of xp[b,k] in direction d          (channel-shared taps)
//   m[b,k]   = sum_d alpha[d,k] h_d[b,k]                    (learnable merger)
//   n[b,k]   = gamma[k] m[b,k] / sqrt(mean_k m[b,k]^2 + eps) (RMS norm over k)
//   y[b,c]   = sum_k U[c,k] n[b,k]                          (back-projection)
//
// Four launches:
// * block_proj_kernel: the projection as a tcgen05 GEMM per 128-pixel tile,
//   D[pixel, k] = sum_c X^T[pixel, c] V^T[c, k], K = C in blocks of 64 channels.
//   X tiles arrive by TMA with the 128-byte swizzle, pixels contiguous (the
//   MN-major operand form); V blocks likewise, channels contiguous (K-major);
//   proxy rows beyond C_proxy are the TMA's zero fill.  The fp32 accumulator
//   lives in tensor memory (two buffers, so the epilogue of one tile overlaps
//   the MMAs of the next) and is written out as xp in fp32.
// * block_taps_kernel: the normalised taps (w0, w2) of every (direction,
//   image, line, position), in scan order.  They are channel-shared, so they
//   are formed once here, one thread each, instead of by every proxy plane's
//   scan (where, one warp per direction, the sigmoids were the scan's
//   critical path).
// * block_scan_kernel: one CTA per proxy plane, one warp per direction; each
//   warp walks its lines, lane t holding P adjacent positions.  It writes h_d
//   in fp32.  The proxy workload is a few planes per image, so this kernel is
//   short and latency bound: each warp stages its inputs (x_proxy, lambda and
//   the taps) in shared memory 8 lines at a time with cp.async, two chunks in
//   flight, so no line waits on memory.
// * block_out_kernel: per 128-pixel tile its prologue merges the four h_d with
//   alpha, normalises over k and writes the bf16 operand n^T (K-major, K =
//   C_proxy padded to 16 or 32) to shared memory; then one tcgen05 MMA per
//   128-channel chunk forms D[c, pixel] = sum_k U[c,k] n[k,pixel] in tensor
//   memory (two buffers), and the epilogue converts it to bf16 and stores it
//   with TMA, each warp its own 32 channel rows.
//
// Every mbarrier wait is bounded; on expiry a warp records the error word at
// offset 0 of the workspace and leaves through its error path.
#include "gspn_internal.h"
#include "gspn_lane.cuh"
#include "gspn_tma.cuh"
#include "gspn_tmem.cuh"

namespace gspn {

namespace {

using namespace lane;

// ---- tcgen05 operand descriptors ------------------------------------------------
using tmem::sdesc;
using tmem::kLayoutNone;
using tmem::kLayoutSw128;
// Instruction descriptor of kind::f16 with bf16 A and B and an fp32
// accumulator: D format bits 4-5, A and B formats bits 7-9 and 10-12, the
// major-ness of A (bit 15) and B (bit 16), N >> 3 at bit 17, M >> 4 at bit 24.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, bool a_mn_major, bool b_mn_major) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn_major ? 1u : 0u) << 15) | ((b_mn_major ? 1u : 0u) << 16) |
           ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}
// D (tensor memory) = A * B^T (+ D when accumulate != 0); issued by one thread
__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// arrive on `bar` once every MMA this thread issued before has completed
__device__ __forceinline__ void mma_commit(uint32_t bar) { tmem::commit(bar); }

// ==================================================================================
// block_proj_kernel: xp = V x, per 128-pixel tile
// ==================================================================================
constexpr int PJ_M = 128;                  // pixels per tile (MMA M)
constexpr int PJ_KB = 64;                  // channels per K block
constexpr int PJ_STAGES = 6;
constexpr int PJ_ABYTES = 2 * 64 * 64 * 2;  // two 64-pixel x 64-channel boxes
constexpr int PJ_THREADS = 192;            // warp 0 TMA, warp 1 MMA, warps 2..5 epilogue

struct ProjArgs {
    float* xp;  // [B][Cp][HW]
    int* err;
    int C, HW, Cp;
    int tiles_per_img, ntiles, nkb;
    uint64_t limit;
};

template <int NPAD>
__host__ __device__ constexpr int pj_stage_bytes() { return PJ_ABYTES + NPAD * 128; }
template <int NPAD>
__host__ __device__ constexpr int pj_smem_bytes() {
    return 1024 + PJ_STAGES * pj_stage_bytes<NPAD>() + 8 * (2 * PJ_STAGES + 5) + 16;
}

template <int NPAD>
__global__ void __launch_bounds__(PJ_THREADS, 1)
    block_proj_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_v,
                      const ProjArgs a) {
    constexpr int SB = pj_stage_bytes<NPAD>();
    static_assert(SB % 1024 == 0, "stages stay 1024-byte aligned for the 128-byte swizzle");
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char* const smem = smem_raw + ((1024u - (tma::smem_u32(smem_raw) & 1023u)) & 1023u);
    const uint32_t sbase = tma::smem_u32(smem);
    const uint32_t full0 = sbase + PJ_STAGES * SB;
    const uint32_t empty0 = full0 + 8 * PJ_STAGES;
    const uint32_t accf0 = empty0 + 8 * PJ_STAGES;  // accumulator buffer ready for the epilogue
    const uint32_t acce0 = accf0 + 16;              // accumulator buffer drained
    const uint32_t fin = acce0 + 16;                // every MMA of this CTA has completed
    uint32_t* const tslot = reinterpret_cast<uint32_t*>(smem + PJ_STAGES * SB + 8 * (2 * PJ_STAGES + 5));
    const int warp = threadIdx.x >> 5, t = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < PJ_STAGES; ++s) {
            tma::mbar_init(full0 + 8 * s, 1);
            tma::mbar_init(empty0 + 8 * s, 1);
        }
        for (int s = 0; s < 2; ++s) {
            tma::mbar_init(accf0 + 8 * s, 1);
            tma::mbar_init(acce0 + 8 * s, 4);
        }
        tma::mbar_init(fin, 1);
        tma::fence_barrier_init();
    }
    if (warp == 1) {
        tmem::alloc(tma::smem_u32(tslot), 64);  // two accumulators of NPAD <= 32 columns
        tmem::relinquish();
    }
    tmem::fence_before();
    __syncthreads();
    tmem::fence_after();
    const uint32_t taddr = *tslot;

    if (warp == 0) {
        // ---- TMA producer: for each tile, nkb blocks of (X: 64 ch x 128 px, V: NPAD x 64 ch)
        if (t == 0) {
            tma::prefetch_map(&tm_x);
            tma::prefetch_map(&tm_v);
            bool ok = true;
            int it = 0;
            for (int tile = blockIdx.x; ok && tile < a.ntiles; tile += gridDim.x) {
                const int b = tile / a.tiles_per_img, pix0 = (tile % a.tiles_per_img) * PJ_M;
                for (int kb = 0; kb < a.nkb; ++kb, ++it) {
                    const int s = it % PJ_STAGES;
                    if (!tma::mbar_wait(empty0 + 8 * s, ((it / PJ_STAGES) & 1) ^ 1, a.limit)) {
                        ok = false;
                        break;
                    }
                    const uint32_t dst = sbase + s * SB, bar = full0 + 8 * s;
                    tma::mbar_expect_tx(bar, SB);
                    tma::load_3d(dst, &tm_x, pix0, kb * PJ_KB, b, bar);
                    tma::load_3d(dst + PJ_ABYTES / 2, &tm_x, pix0 + 64, kb * PJ_KB, b, bar);
                    asm volatile(
                        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
                        " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst + PJ_ABYTES),
                        "l"(reinterpret_cast<uint64_t>(&tm_v)), "r"(kb * PJ_KB), "r"(0), "r"(bar)
                        : "memory");
                }
            }
            if (!ok) atomicExch(a.err, 1);
            // every stage issued has landed before this warp leaves (the MMA
            // warp may have stopped reading them)
            for (int k = it - PJ_STAGES; k < it; ++k)
                if (k >= 0) tma::mbar_wait(full0 + 8 * (k % PJ_STAGES), (k / PJ_STAGES) & 1, 100000000ull);
        }
    } else if (warp == 1) {
        // ---- MMA issuer
        if (t == 0) {
            constexpr uint32_t idesc = idesc_bf16(PJ_M, NPAD, true, false);
            bool ok = true;
            int it = 0, lt = 0;
            for (int tile = blockIdx.x; ok && tile < a.ntiles; tile += gridDim.x, ++lt) {
                const int buf = lt & 1;
                if (!tma::mbar_wait(acce0 + 8 * buf, ((lt >> 1) & 1) ^ 1, a.limit)) {
                    ok = false;
                    break;
                }
                tmem::fence_after();
                const uint32_t d = taddr + (uint32_t)(buf * 32);
                for (int kb = 0; kb < a.nkb; ++kb, ++it) {
                    const int s = it % PJ_STAGES;
                    if (!tma::mbar_wait(full0 + 8 * s, (it / PJ_STAGES) & 1, a.limit)) {
                        ok = false;
                        break;
                    }
                    tmem::fence_after();
                    const uint32_t abase = sbase + s * SB, bbase = abase + PJ_ABYTES;
#pragma unroll
                    for (int kk = 0; kk < PJ_KB / 16; ++kk) {
                        // A: channels 16kk.. = two 8-channel swizzle atoms of 1024 B; the two
                        // 64-pixel halves are 8 KB apart.  B: 32 bytes along each 128-byte row.
                        const uint64_t ad = sdesc(abase + kk * 2048, 8192, 1024, kLayoutSw128);
                        const uint64_t bd = sdesc(bbase + kk * 32, 16, 1024, kLayoutSw128);
                        mma_bf16(d, ad, bd, idesc, (kb | kk) ? 1u : 0u);
                    }
                    mma_commit(empty0 + 8 * s);  // the stage is free once these MMAs have read it
                }
                if (!ok) break;
                mma_commit(accf0 + 8 * buf);
            }
            if (!ok) atomicExch(a.err, 1);
            // no MMA may still run when the tensor memory is released, on any path
            mma_commit(fin);
            tma::mbar_wait(fin, 0, 100000000ull);
        }
        __syncwarp();
    } else {
        // ---- epilogue: warp w reads TMEM lanes 32*(w%4).. = pixels of its quarter
        const int q = warp & 3;
        bool ok = true;
        int lt = 0;
        for (int tile = blockIdx.x; ok && tile < a.ntiles; tile += gridDim.x, ++lt) {
            const int buf = lt & 1;
            ok = __all_sync(FULL, tma::mbar_wait(accf0 + 8 * buf, (lt >> 1) & 1, a.limit));
            if (!ok) break;
            tmem::fence_after();
            uint32_t v[16];
            float r[NPAD];
#pragma unroll
            for (int h = 0; h < NPAD / 16; ++h) {
                tmem::ld_x16(taddr + ((uint32_t)(32 * q) << 16) + (uint32_t)(buf * 32 + 16 * h), v);
                tmem::wait_ld16(v);
#pragma unroll
                for (int i = 0; i < 16; ++i) r[16 * h + i] = __uint_as_float(v[i]);
            }
            tmem::fence_before();
            __syncwarp();
            if (t == 0) tma::mbar_arrive(acce0 + 8 * buf);
            const int b = tile / a.tiles_per_img;
            const int pix = (tile % a.tiles_per_img) * PJ_M + 32 * q + t;
            if (pix < a.HW) {
                float* const o = a.xp + (size_t)b * a.Cp * a.HW + pix;
#pragma unroll
                for (int k = 0; k < NPAD; ++k)
                    if (k < a.Cp) o[(size_t)k * a.HW] = r[k];
            }
        }
        if (!ok && t == 0) atomicExch(a.err, 1);
    }
    tmem::fence_before();
    __syncthreads();
    if (warp == 1) {
        tmem::fence_after();
        tmem::dealloc(taddr, 64);
    }
}

// ==================================================================================
// block_scan_kernel: h_d of every proxy plane, one warp per direction
// ==================================================================================
struct ScanArgs {
    const float* xp;                 // [B][Cp][HW]
    const __nv_bfloat16* lam;        // [4][B][Cp][HW]
    const float2* taps;              // [4][B][line][position]: (w0, w2)
    float* h;                        // [4][B][Cp][HW]
    int B, Cp, H, W, groups;
};

__device__ __forceinline__ float sigm(float z) { return __fdividef(1.f, 1.f + __expf(-z)); }

// taps[((d*B + b)*L + i)*N + j] = (w0, w2) of position j of line i of
// direction d in image b: the sigmoids of the pixel's three tap logits,
// normalised over the taps that exist (w0 = 0 at j = 0, w2 = 0 at j = N-1).
__global__ void __launch_bounds__(256) block_taps_kernel(const __nv_bfloat16* __restrict__ logits,
                                                          float2* __restrict__ taps, int B, int H, int W) {
    const int HW = H * W;
    const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= (int64_t)4 * B * HW) return;
    const int d = (int)(idx / ((int64_t)B * HW));
    const int b = (int)(idx / HW % B);
    const int r = (int)(idx % HW);
    const int N = d < 2 ? W : H;  // positions per line
    const int i = r / N, j = r % N;
    const Walk wk = walk_of(d, H, W);
    const int pix = wk.o + i * wk.si + j * wk.sj;
    const unsigned short* lg = reinterpret_cast<const unsigned short*>(logits) + ((size_t)d * B + b) * 3 * HW;
    const float s0 = j > 0 ? sigm(bf16_bits_to_float(lg[pix])) : 0.f;
    const float s1 = sigm(bf16_bits_to_float(lg[HW + pix]));
    const float s2 = j < N - 1 ? sigm(bf16_bits_to_float(lg[2 * HW + pix])) : 0.f;
    const float rs = __fdividef(1.f, s0 + s1 + s2);
    taps[idx] = make_float2(s0 * rs, s2 * rs);
}

// Inputs of the proxy scans are staged in shared memory a chunk of SC_CH lines
// at a time with cp.async, two chunks per warp in flight, so a line never
// waits for global memory.  Row scans (top->bottom, bottom->top) stage x_proxy
// and lambda of each line as a contiguous row [line][position]; column scans
// (left->right, right->left) stage, for every row, the chunk's SC_CH adjacent
// columns [position][column].  The taps are in scan order already:
// [line][position] in every direction.
constexpr int SC_CH = 8;
// per warp and buffer, for lines of up to nmax positions: xp (fp32), lambda
// (bf16), taps (2 x fp32); sized by the plane so small planes fit more CTAs
__host__ __device__ constexpr int sc_buf_bytes(int nmax) { return SC_CH * nmax * (4 + 2 + 8); }
__host__ __device__ constexpr int sc_smem_bytes(int nmax) { return 4 * 2 * sc_buf_bytes(nmax); }

__device__ __forceinline__ void cp_async16(void* sdst, const void* gsrc) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(tma::smem_u32(sdst)), "l"(gsrc) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

template <int P>
__global__ void __launch_bounds__(128, P <= 2 ? 4 : 1) block_scan_kernel(const ScanArgs a) {
    extern __shared__ __align__(16) unsigned char sc_smem[];
    const int d = threadIdx.x >> 5, t = threadIdx.x & 31;
    const int plane = blockIdx.x;  // b * Cp + k
    const int b = plane / a.Cp;
    const int HW = a.H * a.W;
    const bool rows = d < 2;
    const int L = rows ? a.H : a.W, N = rows ? a.W : a.H;
    const int seg = L / a.groups;
    const Walk wk = walk_of(d, a.H, a.W);
    const float* const xp = a.xp + (size_t)plane * HW;
    const unsigned short* const lam =
        reinterpret_cast<const unsigned short*>(a.lam) + ((size_t)d * a.B * a.Cp + plane) * HW;
    const float2* const tp = a.taps + ((size_t)d * a.B + b) * HW;
    float* const out = a.h + ((size_t)d * a.B * a.Cp + plane) * HW;
    const int sbuf = sc_buf_bytes(a.H > a.W ? a.H : a.W);  // a multiple of 16: H, W are multiples of 8
    unsigned char* const wbuf = sc_smem + d * 2 * sbuf;
    // buffer layout: xp [SC_CH * N] fp32, taps [SC_CH][N] float2, lambda [SC_CH * N] bf16
    const int nch = SC_CH * N;

    // stage chunk c (lines c*SC_CH ..) into buffer c & 1
    auto stage = [&](int c) {
        unsigned char* const bx = wbuf + (c & 1) * sbuf;
        unsigned char* const bt = bx + nch * 4;
        unsigned char* const bl = bt + nch * 8;
        const int i0 = c * SC_CH;
        const int nl = L - i0 < SC_CH ? L - i0 : SC_CH;  // lines in this chunk
        // taps: the chunk's lines are contiguous in scan order, 2 per 16-byte piece
        for (int u = t; u < nl * N / 2; u += 32) cp_async16(bt + u * 16, tp + (size_t)i0 * N + 2 * u);
        if (rows) {
            // line i0 + e is row r: xp N*4 bytes, lambda N*2 bytes, in 16-byte pieces
            const int fx = N / 4, fb = N / 8, per_line = fx + fb;
            for (int u = t; u < nl * per_line; u += 32) {
                const int e = u / per_line, v = u % per_line;
                const int row0 = wk.o + (i0 + e) * wk.si;  // pixel of position 0 of the line
                if (v < fx)
                    cp_async16(bx + (e * N + 4 * v) * 4, xp + row0 + 4 * v);
                else
                    cp_async16(bl + (e * N + 8 * (v - fx)) * 2, lam + row0 + 8 * (v - fx));
            }
        } else {
            // for every row j: the chunk's SC_CH adjacent columns, ascending in the image
            const int c0 = wk.si > 0 ? i0 : a.W - SC_CH - i0;
            for (int u = t; u < N * 3; u += 32) {
                const int j = u / 3, v = u % 3;
                const int pix = j * a.W + c0;
                if (v < 2)
                    cp_async16(bx + (j * SC_CH + 4 * v) * 4, xp + pix + 4 * v);
                else
                    cp_async16(bl + j * SC_CH * 2, lam + pix);
            }
        }
        cp_async_commit();
    };
    // x_proxy (g = 0) or lambda (g = 1) at line e of the chunk, position j
    auto val = [&](const unsigned char* bx, int g, int e, int j) -> float {
        const int idx = rows ? e * N + j : j * SC_CH + (wk.si > 0 ? e : SC_CH - 1 - e);
        if (g == 0) return reinterpret_cast<const float*>(bx)[idx];
        const unsigned short* bl = reinterpret_cast<const unsigned short*>(bx + nch * 12);
        return bf16_bits_to_float(bl[idx]);
    };

    const int nchunks = (L + SC_CH - 1) / SC_CH;
    stage(0);
    if (nchunks > 1) stage(1);
    float h[P];
#pragma unroll
    for (int p = 0; p < P; ++p) h[p] = 0.f;
    int gpos = 0;  // position of the line within its local group
    for (int c = 0; c < nchunks; ++c) {
        if (c + 1 < nchunks)
            cp_async_wait<1>();
        else
            cp_async_wait<0>();
        __syncwarp();  // every lane's pieces of chunk c are in shared memory
        const unsigned char* const bx = wbuf + (c & 1) * sbuf;
        // the chunk's taps and lambda * x first (they do not depend on the
        // state): the sigmoids of all its lines overlap, and the buffer is free
        // to refill before the lines are walked
        float w0c[SC_CH][P], w2c[SC_CH][P], uc[SC_CH][P];
#pragma unroll
        for (int e = 0; e < SC_CH; ++e)
#pragma unroll
            for (int p = 0; p < P; ++p) {
                const int j = P * t + p;
                w0c[e][p] = w2c[e][p] = uc[e][p] = 0.f;
                if (j < N) {
                    uc[e][p] = val(bx, 1, e, j) * val(bx, 0, e, j);
                    const float2 w = reinterpret_cast<const float2*>(bx + nch * 4)[e * N + j];
                    w0c[e][p] = w.x;
                    w2c[e][p] = w.y;
                }
            }
        __syncwarp();  // every lane is done with buffer c & 1 before it is refilled
        if (c + 2 < nchunks) stage(c + 2);
#pragma unroll
        for (int e = 0; e < SC_CH; ++e) {
            const int i = c * SC_CH + e;
            const float left = __shfl_up_sync(FULL, h[P - 1], 1);
            const float right = __shfl_down_sync(FULL, h[0], 1);
            float hn[P];
#pragma unroll
            for (int p = 0; p < P; ++p) {
                // h' = u + w0 h[j-1] + (1 - w0 - w2) h[j] + w2 h[j+1]; h_{-1} = 0 at
                // the start of a scan or of a local group
                const float hl = p == 0 ? left : h[p - 1];
                const float hr = p == P - 1 ? right : h[p + 1];
                hn[p] = gpos == 0 ? uc[e][p] : uc[e][p] + h[p] + w0c[e][p] * (hl - h[p]) + w2c[e][p] * (hr - h[p]);
            }
#pragma unroll
            for (int p = 0; p < P; ++p) {
                const int j = P * t + p;
                h[p] = j < N ? hn[p] : 0.f;
                if (j < N) out[wk.o + i * wk.si + j * wk.sj] = h[p];
            }
            gpos = gpos + 1 == seg ? 0 : gpos + 1;
        }
    }
}

// Named barrier 1 over the 128 prologue/epilogue threads that also ANDs their
// predicates: after a bounded wait every warp learns whether all of them got
// through, so they leave a loop at the same point and none is left waiting
// at a barrier the others will never reach.
__device__ __forceinline__ bool bar_and_128(bool p) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred pi, po;\n\tsetp.ne.u32 pi, %1, 0;\n\t"
        "bar.red.and.pred po, 1, 128, pi;\n\tselp.u32 %0, 1, 0, po;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)p)
        : "memory");
    return r != 0;
}

// ==================================================================================
// block_out_kernel: merge, normalise, project back
// ==================================================================================
constexpr int OB_M = 128;       // channels per chunk (MMA M)
constexpr int OB_N = 128;       // pixels per tile (MMA N)
static_assert(OB_N % 64 == 0 && OB_N <= 128, "whole 64-pixel output boxes; the prologue has 128 threads");
constexpr int OB_THREADS = 160;  // warp 0 MMA, warps 1..4 prologue / epilogue
constexpr int OB_YBUF = OB_M * OB_N * 2;  // one staged output chunk: OB_N / 64 SW128 boxes of 64 pixels

struct OutArgs {
    const float* h;          // [4][B][Cp][HW]
    const float* alpha;      // [4][Cp]
    const float* gamma;      // [Cp]
    const __nv_bfloat16* u;  // [C][Cp]
    int* err;
    int B, C, HW, Cp, norm;
    float eps;
    int tiles_per_img, ntiles, nchunks;
    uint64_t limit;
};

// shared-memory byte offset of element (row, k) of a K-major operand without
// swizzle: 8-row x 16-byte core matrices, K halves 128 B apart, row groups
// KPAD/8 * 128 B apart
template <int KPAD>
__host__ __device__ constexpr uint32_t core_off(int row, int k) {
    return (uint32_t)((row >> 3) * (KPAD / 8) * 128 + (k >> 3) * 128 + (row & 7) * 16 + (k & 7) * 2);
}

template <int KPAD>
__host__ __device__ constexpr int ob_ubytes(int C) { return ((C + OB_M - 1) / OB_M) * OB_M * KPAD * 2; }
template <int KPAD>
__host__ __device__ constexpr int ob_smem_bytes(int C) {
    return 1024 + 2 * OB_YBUF + OB_N * KPAD * 2 + ob_ubytes<KPAD>(C) + 8 * 8 + 16;  // barriers, TMEM slot
}

template <int KPAD>
__global__ void __launch_bounds__(OB_THREADS, 2)
    block_out_kernel(const __grid_constant__ CUtensorMap tm_y, const OutArgs a) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char* const smem = smem_raw + ((1024u - (tma::smem_u32(smem_raw) & 1023u)) & 1023u);
    const uint32_t sbase = tma::smem_u32(smem);
    // [0, 2 YBUF): staged outputs; then the n^T operand; then U; then barriers
    const uint32_t nop = sbase + 2 * OB_YBUF;
    unsigned char* const nopp = smem + 2 * OB_YBUF;
    const uint32_t uop = nop + OB_N * KPAD * 2;
    unsigned char* const uopp = nopp + OB_N * KPAD * 2;
    const int ubytes = ob_ubytes<KPAD>(a.C);
    const uint32_t bars = uop + ubytes;
    const uint32_t accf0 = bars, acce0 = bars + 16, nready = bars + 32, ndone = bars + 40, fin = bars + 48;
    uint32_t* const tslot = reinterpret_cast<uint32_t*>(uopp + ubytes + 64);
    const int warp = threadIdx.x >> 5, t = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < 2; ++s) {
            tma::mbar_init(accf0 + 8 * s, 1);
            tma::mbar_init(acce0 + 8 * s, 4);
        }
        tma::mbar_init(nready, 4);  // the four prologue warps have written n^T
        tma::mbar_init(ndone, 1);   // the MMAs of a tile have read n^T
        tma::mbar_init(fin, 1);     // every MMA of this CTA has completed
        tma::fence_barrier_init();
    }
    // U into its K-major operand layout, zero beyond Cp and beyond C
    for (int e = threadIdx.x; e < ubytes / 2; e += blockDim.x) {
        const int c = e / KPAD, k = e % KPAD;
        const unsigned short v = (c < a.C && k < a.Cp)
                                     ? __ldg(reinterpret_cast<const unsigned short*>(a.u) + (size_t)c * a.Cp + k)
                                     : (unsigned short)0;
        *reinterpret_cast<unsigned short*>(uopp + core_off<KPAD>(c, k)) = v;
    }
    tma::fence_proxy_async();  // the generic writes of U are read by the tensor cores
    if (warp == 0) {
        tmem::alloc(tma::smem_u32(tslot), 2 * OB_N);  // two accumulators of OB_N columns
        tmem::relinquish();
    }
    tmem::fence_before();
    __syncthreads();
    tmem::fence_after();
    const uint32_t taddr = *tslot;

    if (warp == 0) {
        // ---- MMA issuer: per tile, one MMA group per 128-channel chunk
        if (t == 0) {
            constexpr uint32_t idesc = idesc_bf16(OB_M, OB_N, false, false);
            constexpr uint32_t SBO = KPAD / 8 * 128;
            bool ok = true;
            int lt = 0, ch = 0;
            for (int tile = blockIdx.x; ok && tile < a.ntiles; tile += gridDim.x, ++lt) {
                if (!tma::mbar_wait(nready, lt & 1, a.limit)) {
                    ok = false;
                    break;
                }
                tmem::fence_after();
                for (int cb = 0; cb < a.nchunks; ++cb, ++ch) {
                    const int buf = ch & 1;
                    if (!tma::mbar_wait(acce0 + 8 * buf, ((ch >> 1) & 1) ^ 1, a.limit)) {
                        ok = false;
                        break;
                    }
                    tmem::fence_after();
#pragma unroll
                    for (int kk = 0; kk < KPAD / 16; ++kk) {
                        const uint64_t ad = sdesc(uop + cb * (OB_M / 8) * SBO + kk * 256, 128, SBO, kLayoutNone);
                        const uint64_t bd = sdesc(nop + kk * 256, 128, SBO, kLayoutNone);
                        mma_bf16(taddr + (uint32_t)(buf * OB_N), ad, bd, idesc, kk ? 1u : 0u);
                    }
                    mma_commit(accf0 + 8 * buf);
                }
                if (!ok) break;
                mma_commit(ndone);  // n^T may be rewritten once these MMAs are done
            }
            if (!ok) atomicExch(a.err, 1);
            // no MMA may still run when the tensor memory is released, on any path
            mma_commit(fin);
            tma::mbar_wait(fin, 0, 100000000ull);
        }
        __syncwarp();
    } else {
        // ---- prologue + epilogue: thread = pixel (prologue) / channel (epilogue)
        const int q = warp & 3;        // TMEM lane quarter
        const int et = threadIdx.x - 32;  // 0..127
        bool ok = true;
        int lt = 0, ch = 0;
        for (int tile = blockIdx.x; tile < a.ntiles; tile += gridDim.x, ++lt) {
            const int b = tile / a.tiles_per_img, pix0 = (tile % a.tiles_per_img) * OB_N;
            // n^T of the previous tile may still be read by its MMAs; every warp
            // reaches this barrier once per tile, and all leave if one has failed
            ok = bar_and_128(ok && (lt == 0 || tma::mbar_wait(ndone, (lt - 1) & 1, a.limit)));
            if (!ok) break;
            if (et < OB_N) {
                const int pix = pix0 + et;
                float m[KPAD];
#pragma unroll
                for (int k = 0; k < KPAD; ++k) m[k] = 0.f;
                if (pix < a.HW) {
#pragma unroll
                    for (int k = 0; k < KPAD; ++k) {
                        if (k < a.Cp) {
                            float acc = 0.f;
#pragma unroll
                            for (int d = 0; d < 4; ++d)
                                acc = fmaf(__ldg(a.alpha + d * a.Cp + k),
                                           __ldg(a.h + (((size_t)d * a.B + b) * a.Cp + k) * a.HW + pix), acc);
                            m[k] = acc;
                        }
                    }
                    if (a.norm) {
                        float ss = 0.f;
#pragma unroll
                        for (int k = 0; k < KPAD; ++k) ss = fmaf(m[k], m[k], ss);
                        const float r = rsqrtf(ss / (float)a.Cp + a.eps);
#pragma unroll
                        for (int k = 0; k < KPAD; ++k)
                            if (k < a.Cp) m[k] = m[k] * r * __ldg(a.gamma + k);
                    }
                }
#pragma unroll
                for (int k = 0; k < KPAD; k += 8) {
                    uint4 v;
                    v.x = pack_bf2(m[k], m[k + 1]);
                    v.y = pack_bf2(m[k + 2], m[k + 3]);
                    v.z = pack_bf2(m[k + 4], m[k + 5]);
                    v.w = pack_bf2(m[k + 6], m[k + 7]);
                    *reinterpret_cast<uint4*>(nopp + core_off<KPAD>(et, k)) = v;
                }
            }
            // every prologue warp arrives (its lanes wrote their rows of n^T, or none)
            tma::fence_proxy_async();
            __syncwarp();
            if (t == 0) tma::mbar_arrive(nready);
            // epilogue of every 128-channel chunk of this tile: each warp converts
            // and stores its own 32 channel rows (its TMEM lane quarter), so the
            // warps of the CTA do not wait for one another within a tile.  A warp
            // whose wait runs out skips the rest of the tile and all leave
            // together at the next tile's collective barrier.
            for (int cb = 0; cb < a.nchunks; ++cb, ++ch) {
                if (!ok) continue;
                const int buf = ch & 1;
                const bool got = tma::mbar_wait(accf0 + 8 * buf, (ch >> 1) & 1, a.limit);
                // this warp's rows of the chunk staged two chunks ago have been read
                // by its TMA stores
                if (t == 0) tma::bulk_wait_read_n<1>();
                ok = __all_sync(FULL, got);
                if (!ok) continue;
                tmem::fence_after();
                unsigned char* const ys = smem + buf * OB_YBUF;
                const int row = 32 * q + t;  // channel row of the chunk = TMEM lane
                const uint32_t tq = taddr + ((uint32_t)(32 * q) << 16) + (uint32_t)(buf * OB_N);
#pragma unroll
                for (int c64 = 0; c64 < OB_N / 64; ++c64) {
                    // pixels 64 c64 .. +63 of this channel (box c64): two 32-column loads
                    // in flight together; 16-byte chunk j of the 128-byte row at j ^ (row % 8)
                    uint32_t va[32], vb[32];
                    tmem::ld_x32(tq + 64u * c64, va);
                    tmem::ld_x32(tq + 64u * c64 + 32u, vb);
                    tmem::wait_ld(va);
                    tmem::wait_ld(vb);
                    unsigned char* const box = ys + c64 * (OB_M * 128) + row * 128;
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const uint32_t* v = j < 4 ? va + 8 * j : vb + 8 * (j - 4);
                        uint4 w;
                        w.x = pack_bf2(__uint_as_float(v[0]), __uint_as_float(v[1]));
                        w.y = pack_bf2(__uint_as_float(v[2]), __uint_as_float(v[3]));
                        w.z = pack_bf2(__uint_as_float(v[4]), __uint_as_float(v[5]));
                        w.w = pack_bf2(__uint_as_float(v[6]), __uint_as_float(v[7]));
                        *reinterpret_cast<uint4*>(box + ((j ^ (row & 7)) << 4)) = w;
                    }
                }
                tmem::fence_before();
                tma::fence_proxy_async();  // the staged rows are read by TMA stores
                __syncwarp();
                if (t == 0) {
                    tma::mbar_arrive(acce0 + 8 * buf);
                    const int c0 = cb * OB_M + 32 * q;  // first channel of this warp's rows
                    if (c0 < a.C) {
                        const uint32_t ysa = sbase + buf * OB_YBUF + q * 32 * 128;
#pragma unroll
                        for (int c64 = 0; c64 < OB_N / 64; ++c64)
                            if (pix0 + 64 * c64 < a.HW)
                                tma::store_3d(&tm_y, ysa + c64 * OB_M * 128, pix0 + 64 * c64, c0, b);
                    }
                    tma::bulk_commit();
                }
            }
        }
        if (!ok && t == 0) atomicExch(a.err, 1);
        if (t == 0) tma::bulk_wait_all();  // this warp's stores have read shared memory
    }
    tmem::fence_before();
    __syncthreads();
    if (warp == 0) {
        tmem::fence_after();
        tmem::dealloc(taddr, 2 * OB_N);
    }
}

// ---- host side ----------------------------------------------------------------------
bool encode_bf16(CUtensorMap* m, const void* base, int rank, const cuuint64_t* dims, const cuuint64_t* strides,
                 const cuuint32_t* box, CUtensorMapSwizzle swz) {
    EncodeTiledFn fn = encode_tiled();
    if (!fn) return false;
    cuuint32_t es[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(base), dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

struct BlockLayout {
    size_t xp, h, taps, total;
};
BlockLayout block_layout(const gspn_block_desc& d) {
    BlockLayout l;
    const size_t planes = (size_t)d.B * d.Cp * d.H * d.W;
    l.xp = kWsAlign;
    l.h = l.xp + align_up(planes * 4, kWsAlign);
    l.taps = l.h + align_up(4 * planes * 4, kWsAlign);
    l.total = l.taps + align_up((size_t)4 * d.B * d.H * d.W * 8, kWsAlign);
    return l;
}

gspn_status block_validate(const gspn_block_desc* d) {
    if (!d) return GSPN_ERR_INVALID_ARG;
    if (d->B < 1 || d->C < 1 || d->H < 1 || d->W < 1 || d->Cp < 1) return GSPN_ERR_INVALID_ARG;
    if (d->groups < 1 || d->H % d->groups || d->W % d->groups) return GSPN_ERR_INVALID_ARG;
    if (!(d->eps >= 0.f) || d->eps > 1.f) return GSPN_ERR_INVALID_ARG;
    if (d->B > (1 << 20) || d->C > (1 << 20)) return GSPN_ERR_INVALID_ARG;
    // kernel limits: proxy channels, line lengths, 16-byte TMA strides, U in shared memory
    if (d->Cp > 32 || d->H > 128 || d->W > 128) return GSPN_ERR_UNSUPPORTED;
    if (d->C % 8 || d->H % 8 || d->W % 8) return GSPN_ERR_UNSUPPORTED;
    if (d->C > (d->Cp <= 16 ? 3072 : 1536)) return GSPN_ERR_UNSUPPORTED;
    if ((int64_t)d->B * d->C * d->H * d->W > ((int64_t)1 << 40)) return GSPN_ERR_INVALID_ARG;
    if (!encode_tiled()) return GSPN_ERR_UNSUPPORTED;
    return GSPN_OK;
}

template <int NPAD>
gspn_status launch_proj(const DeviceInfo& dev, const gspn_block_desc& d, const void* x, const void* v, float* xp,
                        int* err, cudaStream_t s) {
    const int HW = (int)(d.H * d.W);
    CUtensorMap mx, mv;
    const cuuint64_t xd[3] = {(cuuint64_t)HW, (cuuint64_t)d.C, (cuuint64_t)d.B};
    const cuuint64_t xs[2] = {(cuuint64_t)HW * 2, (cuuint64_t)HW * d.C * 2};
    const cuuint32_t xb[3] = {64, 64, 1};
    const cuuint64_t vd[2] = {(cuuint64_t)d.C, (cuuint64_t)d.Cp};
    const cuuint64_t vs[1] = {(cuuint64_t)d.C * 2};
    const cuuint32_t vb[2] = {64, (cuuint32_t)NPAD};
    if (!encode_bf16(&mx, x, 3, xd, xs, xb, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !encode_bf16(&mv, v, 2, vd, vs, vb, CU_TENSOR_MAP_SWIZZLE_128B))
        return GSPN_ERR_UNSUPPORTED;
    ProjArgs a;
    a.xp = xp;
    a.err = err;
    a.C = (int)d.C;
    a.HW = HW;
    a.Cp = d.Cp;
    a.tiles_per_img = (HW + PJ_M - 1) / PJ_M;
    a.ntiles = (int)d.B * a.tiles_per_img;
    a.nkb = (int)((d.C + PJ_KB - 1) / PJ_KB);
    a.limit = wait_cfg().limit_ns;
    const void* fn = (const void*)block_proj_kernel<NPAD>;
    constexpr int smem = pj_smem_bytes<NPAD>();
    if (ensure_smem_attr(fn, smem, NPAD == 16 ? 32 : 33) != cudaSuccess) return GSPN_ERR_CUDA;
    const int grid = a.ntiles < dev.sm_count ? a.ntiles : dev.sm_count;
    block_proj_kernel<NPAD><<<grid, PJ_THREADS, smem, s>>>(mx, mv, a);
    return cudaGetLastError() == cudaSuccess ? GSPN_OK : GSPN_ERR_CUDA;
}

template <int KPAD>
gspn_status launch_out(const DeviceInfo& dev, const gspn_block_desc& d, const float* h, const float* alpha,
                       const float* gamma, const void* u, void* y, int* err, cudaStream_t s) {
    const int HW = (int)(d.H * d.W);
    CUtensorMap my;
    const cuuint64_t yd[3] = {(cuuint64_t)HW, (cuuint64_t)d.C, (cuuint64_t)d.B};
    const cuuint64_t ys[2] = {(cuuint64_t)HW * 2, (cuuint64_t)HW * d.C * 2};
    const cuuint32_t yb[3] = {64, 32, 1};  // one warp's 32 channel rows of a 64-pixel box
    if (!encode_bf16(&my, y, 3, yd, ys, yb, CU_TENSOR_MAP_SWIZZLE_128B)) return GSPN_ERR_UNSUPPORTED;
    OutArgs a;
    a.h = h;
    a.alpha = alpha;
    a.gamma = gamma;
    a.u = static_cast<const __nv_bfloat16*>(u);
    a.err = err;
    a.B = (int)d.B;
    a.C = (int)d.C;
    a.HW = HW;
    a.Cp = d.Cp;
    a.norm = d.norm ? 1 : 0;
    a.eps = d.eps;
    a.tiles_per_img = (HW + OB_N - 1) / OB_N;
    a.ntiles = (int)d.B * a.tiles_per_img;
    a.nchunks = (int)((d.C + OB_M - 1) / OB_M);
    a.limit = wait_cfg().limit_ns;
    const void* fn = (const void*)block_out_kernel<KPAD>;
    const int smem = ob_smem_bytes<KPAD>((int)d.C);
    if (smem > dev.max_smem_optin) return GSPN_ERR_UNSUPPORTED;
    if (ensure_smem_attr(fn, smem, KPAD == 16 ? 34 : 35) != cudaSuccess) return GSPN_ERR_CUDA;
    // two CTAs per SM where shared memory allows (tensor memory: 2 x 256 columns)
    const int per_sm = 2 * smem <= dev.max_smem_optin ? 2 : 1;
    const int grid = a.ntiles < per_sm * dev.sm_count ? a.ntiles : per_sm * dev.sm_count;
    block_out_kernel<KPAD><<<grid, OB_THREADS, smem, s>>>(my, a);
    return cudaGetLastError() == cudaSuccess ? GSPN_OK : GSPN_ERR_CUDA;
}

}  // namespace

size_t block_workspace(const gspn_block_desc* d) {
    if (block_validate(d) != GSPN_OK) return 0;
    return block_layout(*d).total;
}

gspn_status block_fwd(const gspn_block_desc* d, const void* x, const void* v, const void* logits, const void* lam,
                      const float* alpha, const float* gamma, const void* u, void* y, void* ws, size_t ws_bytes,
                      cudaStream_t s) {
    gspn_status st = block_validate(d);
    if (st != GSPN_OK) return st;
    for (const void* p : {x, v, logits, lam, (const void*)alpha, (const void*)gamma, u, (const void*)y})
        if (!p) return GSPN_ERR_INVALID_ARG;
    for (const void* p : {x, v, logits, lam, (const void*)alpha, (const void*)gamma, u, (const void*)y})
        if (reinterpret_cast<uintptr_t>(p) & 15u) return GSPN_ERR_ALIGNMENT;
    const BlockLayout l = block_layout(*d);
    if (!ws || ws_bytes < l.total) return GSPN_ERR_WORKSPACE;
    if (reinterpret_cast<uintptr_t>(ws) % kWsAlign) return GSPN_ERR_ALIGNMENT;
    DeviceInfo dev;
    if (device_info(&dev) != cudaSuccess) return GSPN_ERR_CUDA;
    char* w = static_cast<char*>(ws);
    int* err = reinterpret_cast<int*>(w);
    float* xp = reinterpret_cast<float*>(w + l.xp);
    float* h = reinterpret_cast<float*>(w + l.h);
    if (cudaMemsetAsync(err, 0, sizeof(int), s) != cudaSuccess) return GSPN_ERR_CUDA;
    st = d->Cp <= 16 ? launch_proj<16>(dev, *d, x, v, xp, err, s) : launch_proj<32>(dev, *d, x, v, xp, err, s);
    if (st != GSPN_OK) return st;
    float2* taps = reinterpret_cast<float2*>(w + l.taps);
    {
        const int64_t n = (int64_t)4 * d->B * d->H * d->W;
        block_taps_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(static_cast<const __nv_bfloat16*>(logits), taps,
                                                                        (int)d->B, (int)d->H, (int)d->W);
        if (cudaGetLastError() != cudaSuccess) return GSPN_ERR_CUDA;
    }
    ScanArgs sa;
    sa.xp = xp;
    sa.lam = static_cast<const __nv_bfloat16*>(lam);
    sa.taps = taps;
    sa.h = h;
    sa.B = (int)d->B;
    sa.Cp = d->Cp;
    sa.H = (int)d->H;
    sa.W = (int)d->W;
    sa.groups = d->groups;
    const int nmax = (int)(d->H > d->W ? d->H : d->W);
    const int grid = (int)d->B * d->Cp;
    const void* sfn = nmax <= 32   ? (const void*)block_scan_kernel<1>
                      : nmax <= 64 ? (const void*)block_scan_kernel<2>
                                   : (const void*)block_scan_kernel<4>;
    const int ssmem = sc_smem_bytes(nmax);
    if (ensure_smem_attr(sfn, ssmem, nmax <= 32 ? 36 : nmax <= 64 ? 37 : 38) != cudaSuccess) return GSPN_ERR_CUDA;
    void* sargs[] = {&sa};
    if (cudaLaunchKernel(sfn, dim3(grid), dim3(128), sargs, ssmem, s) != cudaSuccess) return GSPN_ERR_CUDA;
    if (cudaGetLastError() != cudaSuccess) return GSPN_ERR_CUDA;
    return d->Cp <= 16 ? launch_out<16>(dev, *d, h, alpha, gamma, u, y, err, s)
                       : launch_out<32>(dev, *d, h, alpha, gamma, u, y, err, s);
}

}  // namespace gspn
