// gspn_compact64_bwd.cu -- fast backward for the compact (channel-shared taps)
// four-direction global scan of 64x64 bf16 planes (the 1K foundation shape of
// C-GSPN, "Scaling Parallel Sequence Models to Vision Foundation Models").
//
// The gradient of the line scan ("Parallel Sequence Modeling via Generalized
// Spatial Propagation Network", Key designs 1-2) is its adjoint run from the
// last line to the first ("GSPN-2: Efficient Parallel Sequence Modeling",
// Backward Benchmark: the same kernel-launch design as the forward).  With
// a_i = dL/dh_i, per direction and line:
//   a_i[j]   = G_i[j] + sum_k w_{i+1}[j-k+1][k] a_{i+1}[j-k+1]
//            = G_i[j] + a_{i+1}[j] - p0[j] - p2[j] + p0[j+1] + p2[j-1],
//              p0 = w0 a_{i+1}, p2 = w2 a_{i+1} (weights of line i+1; w1 = 1-w0-w2)
//   dlambda  = x a,   dx += lambda a,
//   dw_k[j]  = a_i[j] h_{i-1}[j+k-1]   (tap products)
// and dlogit_k = w_k (1 - s_k) E_k with E_k = sum over channels of
// (dw_k - sum_m w_m dw_m) (chain rule through w_k = s_k / sum s, s_k =
// sigmoid(logit_k); the taps are channel independent in compact mode).
// Since sum_k w_k E_k = 0, only E_0 and E_2 are summed:
//   E_0 = w_1 (dw_0 - dw_1) + w_2 (dw_0 - dw_2),  E_2 = w_0 (dw_2 - dw_0) + w_1 (dw_2 - dw_1),
//   dlogit_1 = -(1 - s_1) (w_0 E_0 + w_2 E_2).
//
// Design (B200), per plane and per pass (row pass: A = left->right,
// B = right->left over columns s; column pass: A = top->bottom,
// B = bottom->top over rows s):
// * Sweep 1, s ascending: the forward scan of A (h_A) and the adjoint of B
//   (a_B, whose last line is s = 0) both advance with s.  Every step's pair
//   (h_A(s-1), a_B(s)) is parked in tensor memory (TMEM, 512 columns per CTA:
//   each warp owns a 32-lane x 256-column block, lane t = plane columns 2t, 2t+1),
//   so nothing is recomputed and no shared memory is spent on states.
// * Sweep 2, s descending, chunk by chunk: the chunk's states are read back
//   from TMEM, then the chunk is walked backwards running the adjoint of A
//   and the forward of B.  At every
//   s all four of h_A(s-1), a_A(s), h_B(s+1), a_B(s) are at hand, so dlambda
//   of both directions, the pass's share of dx and the tap products of both
//   directions are produced without storing any plane of h or a.
// * dx: the row pass's share goes to a per-warp fp32 plane in the workspace
//   (rewritten for every plane, so it stays in L2); the column pass adds its
//   share and stores dx once.
// * Tap values E_0, E_2: each of the 8 warps of a CTA (8 channels of one
//   image) stores each half chunk of values into its own shared slot; a
//   reducer warp sums the 8 slots and adds the result with bulk
//   shared->global fp32 reduce-adds to L2-resident sums.  Half chunks rotate
//   over three slot sets, each with its own reducer warp, so the reductions
//   overlap and a compute warp rarely waits for a set.
// * x, lambda and dout are streamed by TMA into a per-warp ring of 8-step
//   chunks by four data-producer warps (two compute warps each), so the
//   compute warps issue no copies; the normalised tap weights (a table
//   written by a pre-kernel, one row per scan step with both directions at
//   the same column) by a producer warp into a ring shared by the CTA.
// * 16 warps in four warpgroups: compute (two), then the tap-table producer
//   with the three reducers, then the four data producers.  The helper
//   warpgroups hand registers to the compute ones with setmaxnreg (192 per
//   compute thread, 64 per helper thread).
// * Every wait is bounded (2 s); on expiry the warp records an error word,
//   drains its copies and returns.
#include <atomic>
#include <type_traits>

#include "gspn_internal.h"
#include "gspn_lane.cuh"
#include "gspn_tma.cuh"
#include "gspn_tmem.cuh"

namespace gspn {

namespace {

using namespace lane;

constexpr int S = 64;           // H = W
constexpr int LPL = 32;         // lanes per line, 2 positions each
constexpr int NCW = 8;          // consumer warps (one plane each)
constexpr int NST = 2;          // data ring stages per warp
constexpr int NWS = 4;          // weight ring stages per CTA
constexpr int BOX = 1024;       // one plane of one tensor per chunk
constexpr int STAGE = 4 * BOX;  // x, lambda_A, lambda_B, dout
constexpr int WCHUNK = 8 * S * 16;
constexpr int DSLOT = 4 * 4 * S * 4;      // one warp's tap values of half a chunk: [step][dir*2 + value][position j]
constexpr int WARP_BYTES = NST * STAGE;   // data ring per warp
constexpr int WRING = NCW * WARP_BYTES;
constexpr int DSTG = WRING + NWS * WCHUNK;    // 2 sets x NCW slots
constexpr int NSET = 3;                         // slot sets, one reducer warp each
constexpr int DOUT = DSTG + NSET * NCW * DSLOT;  // a reduced half chunk per set: [dir*2 + value][step][position j]
constexpr int DLS = DOUT + NSET * DSLOT;          // per warp: row-pass dlambda of a chunk, A then B, [row % 2][row / 2][8 columns]
constexpr int BARS = DLS + NCW * 2 * BOX;
constexpr int NBAR = 2 * NCW * NST + 2 * NWS + 2 * NSET + 1;
constexpr int SMEM_BYTES = 1024 + BARS + 8 * NBAR + 16;  // + the TMEM address
constexpr int CHUNKS_PER_GROUP = 32;  // row pass sweeps 1, 2; column pass sweeps 1, 2 (8 chunks each)
constexpr int NDP = NCW / 2;                     // data producers, two compute warps each
// warpgroups 0, 1: compute warps; warpgroup 2: tap-table producer and the
// tap-value reducers; warpgroup 3: the data producers
constexpr int THREADS = (NCW + 1 + NSET + NDP) * 32;
static_assert(THREADS == 512, "four warpgroups");
// Launched at 128 registers per thread (65536 / 512).  The helper warpgroups
// give registers up and the compute warpgroups take them: on each scheduler
// (warps k, k+4, k+8, k+12) 2 x 32 x kComputeRegs + 2 x 32 x kHelperRegs
// must equal its 16384, or a setmaxnreg.inc would wait forever.
constexpr int kComputeRegs = 192, kHelperRegs = 64;
static_assert(2 * 32 * kComputeRegs + 2 * 32 * kHelperRegs == 16384, "register split");
static_assert(SMEM_BYTES <= 232448, "shared memory budget");

// ---- backward tap table ---------------------------------------------------------------
// Row (b, pass, s) of the table holds the taps of both directions' lines at
// column (row pass) or row (column pass) s, as pairs over the positions
// j = 2t, 2t+1 of lane t: float4 t = (w0_A, w0_A', w2_A, w2_A') and float4
// 32 + t = (w0_B, w0_B', w2_B, w2_B') (' = position 2t+1).  Pass 0: A =
// left->right (slot 2), B = right->left (slot 3), pixel (j, s); pass 1: A =
// top->bottom (slot 0), B = bottom->top (slot 1), pixel (s, j).
template <typename T>
__device__ __forceinline__ void gate_w(const T* lg, int pix, int j, float* w0, float* w2) {
    const float s0 = j > 0 ? sigmoidf(load_elt(lg, pix)) : 0.f;
    const float s1 = sigmoidf(load_elt(lg, S * S + pix));
    const float s2 = j < S - 1 ? sigmoidf(load_elt(lg, 2 * S * S + pix)) : 0.f;
    const float r = 1.f / (s0 + s1 + s2);
    *w0 = s0 * r;
    *w2 = s2 * r;
}

template <typename T>
__global__ void c64b_table_kernel(const T* __restrict__ logits, float4* __restrict__ btab, float* __restrict__ dsum,
                                  int* err, int B) {
    const int idx = blockIdx.x * blockDim.x + threadIdx.x;
    if (idx == 0) *err = 0;
    const int n = B * 2 * S * LPL;  // one thread per (b, pass, s, lane)
    // the tap sums start at zero: 2 directions x 2 values per pixel of each pass
    for (int q = idx; q < n * 8; q += gridDim.x * blockDim.x) dsum[q] = 0.f;
    if (idx >= n) return;
    const int t = idx & 31, s = (idx >> 5) & 63, pass = (idx >> 11) & 1, b = idx >> 12;
    const int slotA = pass ? 0 : 2, slotB = pass ? 1 : 3;
    float w[2][2][2];  // [dir][position][w0, w2]
    for (int p = 0; p < 2; ++p) {
        const int j = 2 * t + p, pix = pass ? s * S + j : j * S + s;
        gate_w(logits + (size_t)(slotA * B + b) * 3 * S * S, pix, j, &w[0][p][0], &w[0][p][1]);
        gate_w(logits + (size_t)(slotB * B + b) * 3 * S * S, pix, j, &w[1][p][0], &w[1][p][1]);
    }
    float4* row = btab + ((size_t)(b * 2 + pass) * S + s) * S;
    row[t] = make_float4(w[0][0][0], w[0][1][0], w[0][0][1], w[0][1][1]);
    row[LPL + t] = make_float4(w[1][0][0], w[1][1][0], w[1][0][1], w[1][1][1]);
}

// dlogits from the tap sums: with the pixel's sigmoids s_k and normalised
// weights w_k over its valid taps, dlogit_0 = w_0 (1 - s_0) E_0,
// dlogit_2 = w_2 (1 - s_2) E_2, dlogit_1 = -(1 - s_1) (w_0 E_0 + w_2 E_2); zero on
// the first line of each direction (its taps are never used) and on invalid taps.
template <typename T>
__global__ void c64b_dlogits_kernel(const T* __restrict__ logits, const float* __restrict__ dsum,
                                    T* __restrict__ dlogits, int B) {
    const int idx = blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= 4 * B * S * S) return;
    const int pix = idx & (S * S - 1), b = (idx >> 12) % B, slot = (idx >> 12) / B;
    const int r = pix >> 6, c = pix & 63;
    const int pass = slot < 2 ? 1 : 0, dir = slot & 1;  // dir 0 = A, 1 = B
    // scan coordinates: row pass (s = column, j = row), column pass (s = row, j = column)
    const int s = pass ? r : c, j = pass ? c : r;
    const bool first_line = dir == 0 ? s == 0 : s == S - 1;
    const T* lg = logits + (size_t)(slot * B + b) * 3 * S * S;
    T* out = dlogits + (size_t)(slot * B + b) * 3 * S * S;
    const bool v0 = j > 0, v2 = j < S - 1;
    const float s0 = v0 ? sigmoidf(load_elt(lg, pix)) : 0.f;
    const float s1 = sigmoidf(load_elt(lg, S * S + pix));
    const float s2 = v2 ? sigmoidf(load_elt(lg, 2 * S * S + pix)) : 0.f;
    const float rs = 1.f / (s0 + s1 + s2);
    const float w0 = s0 * rs, w2 = s2 * rs;
    const size_t base = (((size_t)(b * 2 + pass) * 4 + dir * 2) * S + s) * S + j;
    const float e0 = first_line ? 0.f : dsum[base];
    const float e2 = first_line ? 0.f : dsum[base + (size_t)S * S];
    store_elt(out, pix, v0 ? w0 * (1.f - s0) * e0 : 0.f);
    store_elt(out, (size_t)S * S + pix, -(1.f - s1) * (w0 * e0 + w2 * e2));
    store_elt(out, (size_t)2 * S * S + pix, v2 ? w2 * (1.f - s2) * e2 : 0.f);
}

struct C64BArgs {
    const float4* btab;
    float* dsum;  // [B][pass][dir*2 + value][s][j]: E_0, E_2 sums
    float* dxh;   // per-warp fp32 planes: the row pass's share of dx
    __nv_bfloat16* dx;
    __nv_bfloat16* dlam;
    int* err;
    int B, C;
    int groups;   // B * C / 8
    int segmask;  // local groups: lines per group - 1 (a power of two minus one; 63 = global)
    uint64_t limit;  // bound of every wait on data, a stage or another warp (ns)
    int stall;       // test hook: compute warp 0 of CTA 0 first waits on a barrier nothing completes
};

// bf16 element e of 8 packed in a uint4, widened
__device__ __forceinline__ float bfv(const uint4& v, int e) {
    const uint32_t w = word_of(v, e >> 1);
    return (e & 1) ? __uint_as_float(w & 0xffff0000u) : __uint_as_float(w << 16);
}
// the two bf16 halves of a word, widened: (low, high)
__device__ __forceinline__ float2 bf2(uint32_t w) {
    return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}

// Lane t holds positions j = 2t, 2t+1 of a line as a float2; all arithmetic
// below is packed over the pair.
__device__ __forceinline__ float2 add2(float2 a, float2 b) { return __fadd2_rn(a, b); }
__device__ __forceinline__ float2 mul2(float2 a, float2 b) { return __fmul2_rn(a, b); }
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }

// Tap weights of a line for this lane's pair of positions.
struct Taps {
    float2 w0, w2;
};

// Neighbour mix of the previous state h: m[j] = sum_k w_k[j] h[j+k-1],
// written as h + w2 (hR - h) + w0 (hL - h) with w1 = 1 - w0 - w2; hL, hR
// are h shifted by one position.  The shuffles rotate, so lane 0 reads
// position 63 as its left neighbour and lane 31 position 0 as its right
// one: both meet a zero tap weight (w0 at j = 0, w2 at j = 63).
__device__ __forceinline__ float2 mix(float2 h, const Taps& w, int t, float2& hL, float2& hR) {
    hL = make_float2(__shfl_sync(FULL, h.y, (t + 31) & 31), h.x);
    hR = make_float2(h.y, __shfl_sync(FULL, h.x, (t + 1) & 31));
    return fma2(w.w0, sub2(hL, h), fma2(w.w2, sub2(hR, h), h));
}

// Forward step h' = w0 hL + w1 h + w2 hR + lx written so that only two FMAs
// follow the shuffles (w1 h + lx is formed while they are in flight); m =
// h' - lx is the neighbour mix, for the tap values.
__device__ __forceinline__ float2 fwd_step(float2 h, float2 lx, const Taps& w, int t, float2& hL, float2& hR,
                                           float2& m) {
    hL = make_float2(__shfl_sync(FULL, h.y, (t + 31) & 31), h.x);
    hR = make_float2(h.y, __shfl_sync(FULL, h.x, (t + 1) & 31));
    const float2 w1 = sub2(sub2(make_float2(1.f, 1.f), w.w0), w.w2);
    const float2 hn = fma2(w.w2, hR, fma2(w.w0, hL, fma2(w1, h, lx)));
    m = sub2(hn, lx);
    return hn;
}

// Adjoint step: a(line i) = g + W_{i+1}^T a(line i+1), with w the taps of
// line i+1: a'[j] = g[j] + w1[j] a[j] + w0[j+1] a[j+1] + w2[j-1] a[j-1].  The
// rotated shuffles bring in w0 a at j = 0 and w2 a at j = 63, both zero.
// g + a arrives already formed (from the bf16 g by one mixed-precision FMA per
// position: g * 1 + a, a single rounding); the in-lane terms are summed while
// the shuffles are in flight.
__device__ __forceinline__ float2 adjoint_ga(float2 a, float2 ga, const Taps& w, int t) {
    const float2 p0 = mul2(w.w0, a), p2 = mul2(w.w2, a);
    const float p0r = __shfl_sync(FULL, p0.x, (t + 1) & 31);
    const float p2l = __shfl_sync(FULL, p2.y, (t + 31) & 31);
    const float2 n = add2(fma2(make_float2(-1.f, -1.f), p2, fma2(make_float2(-1.f, -1.f), p0, ga)),
                          make_float2(p0.y, p2.x));
    return add2(n, make_float2(p2l, p0r));
}
constexpr uint32_t kOneBf2 = 0x3F803F80u;  // bf16 1.0 in both halves

// 16 warps, 4 per scheduler; see kComputeRegs for the register split
template <bool LOCAL>
__global__ void __launch_bounds__(THREADS, 1)
    c64b_kernel(const __grid_constant__ CUtensorMap tm_xc, const __grid_constant__ CUtensorMap tm_lc,
                const __grid_constant__ CUtensorMap tm_gc, const __grid_constant__ CUtensorMap tm_xr,
                const __grid_constant__ CUtensorMap tm_lr, const __grid_constant__ CUtensorMap tm_gr,
                const __grid_constant__ CUtensorMap tm_dl, const C64BArgs a) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char* const smem = smem_raw + ((1024u - (tma::smem_u32(smem_raw) & 1023u)) & 1023u);
    const uint32_t sbase = tma::smem_u32(smem);
    const int warp = threadIdx.x >> 5, t = threadIdx.x & 31;
    const uint32_t wfull0 = sbase + BARS + 8 * NCW * NST;
    const uint32_t wempty0 = wfull0 + 8 * NWS;
    const uint32_t dfull0 = wempty0 + 8 * NWS;  // [set]: the compute warps' slots of a chunk are written
    const uint32_t dempty0 = dfull0 + 8 * NSET;  // [set]: the reducer has read the set
    const uint32_t done0 = dempty0 + 8 * NSET;   // every compute warp is done with the tensor memory
    const uint32_t xempty0 = done0 + 8;          // [warp][stage]: the compute warp has read its data stage
    uint32_t* const tslot = reinterpret_cast<uint32_t*>(smem + BARS + 8 * NBAR);
    if ((int)blockIdx.x >= a.groups) return;

    if (threadIdx.x == 0) {
        for (int s = 0; s < NCW * NST; ++s) tma::mbar_init(sbase + BARS + 8 * s, 1);
        for (int s = 0; s < NWS; ++s) {
            tma::mbar_init(wfull0 + 8 * s, 1);
            tma::mbar_init(wempty0 + 8 * s, NCW);
        }
        for (int s = 0; s < NSET; ++s) {
            tma::mbar_init(dfull0 + 8 * s, NCW * 32);
            tma::mbar_init(dempty0 + 8 * s, 1);
        }
        tma::mbar_init(done0, NCW);
        for (int s = 0; s < NCW * NST; ++s) tma::mbar_init(xempty0 + 8 * s, 32);
        tma::fence_barrier_init();
    }
    if (warp == 0) {  // compute warp 0 owns the CTA's tensor memory: all 512 columns
        tmem::alloc(tma::smem_u32(tslot), 512);
        tmem::relinquish();
    }
    tmem::fence_before();
    __syncthreads();
    tmem::fence_after();
    const uint32_t taddr = *tslot;

    const int ngroups_here = (a.groups - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x;
    const int nchunks = ngroups_here * CHUNKS_PER_GROUP;
    const int BC = a.B * a.C;

    // chunk kk of the CTA sequence: pass, sweep, chunk index q of 8 steps
    auto chunk_info = [](int kk, int& pass, int& sweep, int& q) {
        const int l = kk % CHUNKS_PER_GROUP;
        pass = l >> 4;
        sweep = (l >> 3) & 1;
        q = sweep ? 7 - (l & 7) : (l & 7);
    };

    // ---------------- helper warpgroups 2 and 3 ----------------
    // Every helper warp executes the one register release below (a warpgroup
    // must execute the same setmaxnreg), then takes its role.
    if (warp >= NCW) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kHelperRegs) : "memory");
    // ---------------- producer warp: tap-table chunks ----------------
    if (warp == NCW) {
        if (t == 0) {
            for (int kc = 0; kc < nchunks; ++kc) {
                const int ws = kc % NWS;
                if (!tma::mbar_wait_sleep(wempty0 + 8 * ws, ((kc / NWS) & 1) ^ 1, 200, a.limit)) {
                    atomicExch(a.err, 1);
                    break;
                }
                const int group = (int)blockIdx.x + (kc / CHUNKS_PER_GROUP) * (int)gridDim.x;
                const int b = (8 * group) / a.C;
                int pass, sweep, q;
                chunk_info(kc, pass, sweep, q);
                const float4* src = a.btab + ((size_t)(b * 2 + pass) * S + 8 * q) * S;
                tma::mbar_expect_tx(wfull0 + 8 * ws, WCHUNK);
                tma::load_1d(sbase + WRING + ws * WCHUNK, src, WCHUNK, wfull0 + 8 * ws);
            }
        }
        return;
    }

    // ---------------- reducer warps: tap values of each sweep-2 half chunk ----------------
    // Half chunk n of the CTA (pass-major within a group, q descending, the upper
    // 4 steps of a chunk first) sits in slot set n % NSET, which reducer warp
    // n % NSET owns.  It sums the 8 slots into its reduced buffer, hands the set
    // back, and adds the half chunk to the image's sums (rows 8q+4h..8q+4h+3 of
    // each of the 4 [s][j] planes) by 4 bulk reduce-adds of 1 KB.
    if (warp >= NCW + 1 && warp < NCW + 1 + NSET) {
        // reducer rid takes the pieces of slot set rid (every NSET-th half chunk)
        const int rid = warp - (NCW + 1);
        const float4* const sets = reinterpret_cast<const float4*>(smem + DSTG);
        int n = 0;
        bool ok = true;
        for (int group = blockIdx.x; ok && group < a.groups; group += gridDim.x) {
            const int b = (8 * group) / a.C;
            for (int l = 0; l < 32; ++l, ++n) {
                const int pass = l >> 4, q = 7 - ((l >> 1) & 7), h = 1 - (l & 1), set = n % NSET;
                if (set != rid) continue;
                float* const dsum = a.dsum + (size_t)(b * 2 + pass) * 4 * S * S + (8 * q + 4 * h) * S;
                if (!__all_sync(FULL, tma::mbar_wait_sleep(dfull0 + 8 * set, (n / NSET) & 1, 128, a.limit))) {
                    ok = false;
                    break;
                }
                if (t == 0) tma::bulk_wait_read();  // this reducer's previous reduces have read its buffer
                __syncwarp();
                const float4* const src = sets + set * NCW * (DSLOT / 16);
                float4* const outp = reinterpret_cast<float4*>(smem + DOUT + set * DSLOT);
#pragma unroll 4
                for (int i = 0; i < DSLOT / 16 / 32; ++i) {
                    const int f = i * 32 + t;  // float4 f of a slot: step f >> 6, row (f >> 4) & 3, j = 4 (f & 15)
                    float4 acc = src[f];
#pragma unroll
                    for (int w = 1; w < NCW; ++w) {
                        const float4 v = src[w * (DSLOT / 16) + f];
                        acc.x += v.x;
                        acc.y += v.y;
                        acc.z += v.z;
                        acc.w += v.w;
                    }
                    outp[(((f >> 4) & 3) * 4 + (f >> 6)) * 16 + (f & 15)] = acc;
                }
                __syncwarp();
                if (t == 0) tma::mbar_arrive(dempty0 + 8 * set);
                tma::fence_proxy_async();
                __syncwarp();
                if (t == 0) {
                    for (int r = 0; r < 4; ++r)
                        tma::reduce_add_f32(dsum + (size_t)r * S * S, sbase + DOUT + set * DSLOT + r * 1024, 1024);
                    tma::bulk_commit();
                }
            }
        }
        if (t == 0) {
            if (!ok) atomicExch(a.err, 1);
            tma::bulk_wait_all();
        }
        return;
    }

    // ---------------- data producers ----------------
    // Lane 0 of producer p streams the data chunks of compute warps 2p and 2p+1:
    // chunk kk of warp w (plane 8*group + w of group blockIdx.x + (kk/32)*gridDim.x)
    // is x, lambda_A, lambda_B (sweep 2 only) and dout of the chunk's 8 columns
    // (row pass: [row % 2][row / 2][8 columns] through the 4-D view) or rows
    // (column pass: [8 rows][64 columns]), into stage kk % NST of the warp's
    // ring once the warp has read what the stage held.  The compute warps
    // issue no copies themselves: issuing them took a fifth of their time.
    if (warp >= NCW + 1 + NSET) {
        if (t == 0) {
            const int pw = warp - (NCW + 1 + NSET);
            if (pw == 0) {
                tma::prefetch_map(&tm_xc);
                tma::prefetch_map(&tm_lc);
                tma::prefetch_map(&tm_gc);
                tma::prefetch_map(&tm_xr);
                tma::prefetch_map(&tm_lr);
                tma::prefetch_map(&tm_gr);
            }
            bool ok = true;
            for (int kk = 0; ok && kk < nchunks; ++kk) {
                const int group = (int)blockIdx.x + (kk / CHUNKS_PER_GROUP) * (int)gridDim.x;
                int pass, sweep, q;
                chunk_info(kk, pass, sweep, q);
                const int st = kk % NST;
                const int la = pass ? 0 : 2, lb = pass ? 1 : 3;  // lambda slots of A and B
                for (int w = 2 * pw; w < 2 * pw + 2; ++w) {
                    if (!tma::mbar_wait(xempty0 + 8 * (w * NST + st), ((kk / NST) & 1) ^ 1, a.limit)) {
                        ok = false;
                        break;
                    }
                    const int plane = 8 * group + w;
                    const uint32_t dst = sbase + w * WARP_BYTES + st * STAGE;
                    const uint32_t bar = sbase + BARS + 8 * (w * NST + st);
                    tma::mbar_expect_tx(bar, sweep ? 4 * BOX : 3 * BOX);
                    if (pass == 0) {
                        tma::load_4d(dst + 0 * BOX, &tm_xc, 8 * q, 0, 0, plane, bar);
                        tma::load_4d(dst + 1 * BOX, &tm_lc, 8 * q, 0, 0, la * BC + plane, bar);
                        if (sweep) tma::load_4d(dst + 2 * BOX, &tm_lc, 8 * q, 0, 0, lb * BC + plane, bar);
                        tma::load_4d(dst + 3 * BOX, &tm_gc, 8 * q, 0, 0, plane, bar);
                    } else {
                        tma::load_3d(dst + 0 * BOX, &tm_xr, 0, 8 * q, plane, bar);
                        tma::load_3d(dst + 1 * BOX, &tm_lr, 0, 8 * q, la * BC + plane, bar);
                        if (sweep) tma::load_3d(dst + 2 * BOX, &tm_lr, 0, 8 * q, lb * BC + plane, bar);
                        tma::load_3d(dst + 3 * BOX, &tm_gr, 0, 8 * q, plane, bar);
                    }
                }
            }
            if (!ok) atomicExch(a.err, 1);
        }
        return;
    }
    return;
    }  // helper warpgroups

    // ---------------- consumer warps ----------------
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kComputeRegs) : "memory");
    unsigned char* const ringp = smem + warp * WARP_BYTES;
    float* const dxslot = a.dxh + ((size_t)blockIdx.x * NCW + warp) * S * S;
    // sweep-1 states of this warp's plane: lane t of TMEM quarter warp % 4,
    // columns 256 * (warp / 4) + 4s .. +3 = (h_A(s-1), a_B(s)) at positions 2t, 2t+1
    const uint32_t tstate = taddr + ((uint32_t)(32 * (warp & 3)) << 16) + 256u * (uint32_t)(warp >> 2);
    unsigned char* const dlst = smem + DLS + warp * 2 * BOX;
    const uint32_t dlsa = sbase + DLS + warp * 2 * BOX;
    const uint64_t keep = l2_evict_last_policy();
    const unsigned char* const wring = smem + WRING;
    const uint32_t bar0 = sbase + BARS + 8 * NST * warp;

    if (t == 0) tma::prefetch_map(&tm_dl);

    int k = 0, stage = 0;
    uint32_t phase = 0;
    auto fail = [&]() {
        if (t == 0) atomicExch(a.err, 1);
        tmem::wait_st();  // no TMEM store may outlive the warp
        for (int kk = k; kk < k + NST && kk < nchunks; ++kk)
            tma::mbar_wait(bar0 + 8 * (kk % NST), (kk / NST) & 1, 100000000ull);
        for (int kk = k; kk < k + NWS && kk < nchunks; ++kk)
            tma::mbar_wait(wfull0 + 8 * (kk % NWS), (kk / NWS) & 1, 100000000ull);
    };
    auto acquire = [&]() -> bool {
        const bool ok1 = tma::mbar_wait(bar0 + 8 * stage, (phase >> stage) & 1u, a.limit);
        const bool ok2 = tma::mbar_wait(wfull0 + 8 * (k % NWS), (k / NWS) & 1, a.limit);
        return __all_sync(FULL, ok1 && ok2);
    };
    // the data stage is in registers: hand it back to its producer (every lane
    // orders its reads of the stage before the async-proxy refill with a proxy
    // fence of its own, then arrives)
    auto release_data = [&]() {
        tma::fence_proxy_async();
        tma::mbar_arrive(xempty0 + 8 * (warp * NST + stage));
        phase ^= 1u << stage;
        stage = stage == NST - 1 ? 0 : stage + 1;
    };
    // done with the weight stage of chunk k
    auto release_w = [&]() {
        tma::fence_proxy_async();
        __syncwarp();
        if (t == 0) tma::mbar_arrive(wempty0 + 8 * (k % NWS));
        ++k;
    };
    // tap weights of row e of the current weight stage (line 8q+e of both directions)
    auto wrow = [&](int e, Taps& A, Taps& Bt) {
        const unsigned char* src = wring + (k % NWS) * WCHUNK + e * 1024 + t * 16;
        const float4 va = lds128f(src), vb = lds128f(src + 512);
        A.w0 = make_float2(va.x, va.y);
        A.w2 = make_float2(va.z, va.w);
        Bt.w0 = make_float2(vb.x, vb.y);
        Bt.w2 = make_float2(vb.z, vb.w);
    };
    // tap values of sweep-2 half chunk number dchunk: this warp's slot in set
    // dchunk % NSET, free once the reducer has handed the set back
    int dchunk = 0;
    auto dslot = [&]() -> float* {
        const bool ok = tma::mbar_wait(dempty0 + 8 * (dchunk % NSET), ((dchunk / NSET) & 1) ^ 1, a.limit);
        if (!__all_sync(FULL, ok)) return nullptr;
        return reinterpret_cast<float*>(smem + DSTG + ((dchunk % NSET) * NCW + warp) * DSLOT);
    };
    auto dpublish = [&]() {
        tma::mbar_arrive(dfull0 + 8 * (dchunk % NSET));  // every lane: its stores are released
        ++dchunk;
    };

    bool stalled = false;
    if (a.stall && blockIdx.x == 0 && warp == 0 &&
        !__all_sync(FULL, tma::mbar_wait(done0, 0, a.limit))) {
        // test hook: phase 0 of done0 needs this warp's own final arrival, so the
        // wait above can only run out; take the error path
        fail();
        stalled = true;
    }
    for (int group = blockIdx.x; !stalled && group < a.groups; group += gridDim.x) {
        const int plane = 8 * group + warp;

        auto run_pass = [&](auto pass_c) -> bool {
            constexpr int pass = decltype(pass_c)::value;
            const int la = pass ? 0 : 2, lb = pass ? 1 : 3;
            __nv_bfloat16* const dlamA = a.dlam + ((size_t)la * BC + plane) * S * S;
            __nv_bfloat16* const dlamB = a.dlam + ((size_t)lb * BC + plane) * S * S;
            const Taps zero_taps = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};

            // ---------------- sweep 1: h_A forward and a_B adjoint, s ascending ----------------
            float2 hA = make_float2(0.f, 0.f), aB = make_float2(0.f, 0.f);
            Taps WBp = zero_taps;  // B taps of line s-1 (none before s = 0: a_B(-1) = 0)
            for (int q = 0; q < 8; ++q) {
                uint32_t sv[32];  // (h_A(s-1), a_B(s)) of the chunk's 8 steps, for TMEM
                if (!acquire()) { fail(); return false; }
                uint4 X[2] = {}, LA[2] = {}, G[2] = {};
                uint32_t Xr[8] = {}, LAr[8] = {}, Gr[8] = {};
                if constexpr (pass == 0) {
                    const unsigned char* st = ringp + stage * STAGE + t * 16;  // rows 2t, 2t+1: slices 0, 1
#pragma unroll
                    for (int p = 0; p < 2; ++p) {
                        X[p] = lds128(st + 0 * BOX + p * 512);
                        LA[p] = lds128(st + 1 * BOX + p * 512);
                        G[p] = lds128(st + 3 * BOX + p * 512);
                    }
                } else {
                    const unsigned char* st = ringp + stage * STAGE + t * 4;
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        Xr[e] = lds32(st + 0 * BOX + e * 128);
                        LAr[e] = lds32(st + 1 * BOX + e * 128);
                        Gr[e] = lds32(st + 3 * BOX + e * 128);
                    }
                }
                release_data();
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    Taps WA, WB;
                    wrow(e, WA, WB);
                    // lambda x and g + a_B from the bf16 words by mixed-precision FMAs
                    float2 lx, ga;
                    if constexpr (pass == 0) {
                        lx = make_float2(fma_bf(e & 1, word_of(LA[0], e >> 1), word_of(X[0], e >> 1), 0.f),
                                         fma_bf(e & 1, word_of(LA[1], e >> 1), word_of(X[1], e >> 1), 0.f));
                    } else {
                        lx = make_float2(fma_bf_lo(LAr[e], Xr[e], 0.f), fma_bf_hi(LAr[e], Xr[e], 0.f));
                    }
                    float2 hL, hR;
                    // local groups: line s of A starts a group, and line s-1 of B (the
                    // next in B's order) starts one, exactly when s is a multiple of seg
                    if (LOCAL && ((8 * q + e) & a.segmask) == 0) {
                        hA = make_float2(0.f, 0.f);
                        aB = make_float2(0.f, 0.f);
                    }
                    sv[4 * e] = __float_as_uint(hA.x);
                    sv[4 * e + 1] = __float_as_uint(hA.y);
                    float2 mA_;
                    hA = fwd_step(hA, lx, WA, t, hL, hR, mA_);
                    if constexpr (pass == 0) {
                        ga = make_float2(fma_bf(e & 1, word_of(G[0], e >> 1), kOneBf2, aB.x),
                                         fma_bf(e & 1, word_of(G[1], e >> 1), kOneBf2, aB.y));
                    } else {
                        ga = make_float2(fma_bf_lo(Gr[e], kOneBf2, aB.x), fma_bf_hi(Gr[e], kOneBf2, aB.y));
                    }
                    aB = adjoint_ga(aB, ga, WBp, t);
                    sv[4 * e + 2] = __float_as_uint(aB.x);
                    sv[4 * e + 3] = __float_as_uint(aB.y);
                    WBp = WB;
                }
                tmem::st_x32(tstate + 32 * q, sv);
                release_w();
            }
            tmem::wait_st();  // sweep 2 reads what sweep 1 stored

            // ---------------- sweep 2: s descending ----------------
            float2 aA = make_float2(0.f, 0.f), hB = make_float2(0.f, 0.f);
            Taps WAn = zero_taps;  // A taps of line s+1 (none after s = 63: a_A(64) = 0)
            for (int qq = 0; qq < 8; ++qq) {
                const int q = 7 - qq;
                // column pass: the row pass's dx share of columns 2t, 2t+1, rows 8q..8q+7
                // (loaded early; the scratch plane is column-major)
                float4 dxc[2][2];
                if constexpr (pass == 1) {
#pragma unroll
                    for (int p = 0; p < 2; ++p)
#pragma unroll
                        for (int h = 0; h < 2; ++h) dxc[p][h] = ldg128_keep(dxslot + (2 * t + p) * S + 8 * q + 4 * h, keep);
                }
                if (!acquire()) { fail(); return false; }
                uint4 X[2] = {}, LA[2] = {}, LB[2] = {}, G[2] = {};
                uint32_t Xr[8] = {}, LAr[8] = {}, LBr[8] = {}, Gr[8] = {};
                if constexpr (pass == 0) {
                    const unsigned char* st = ringp + stage * STAGE + t * 16;  // rows 2t, 2t+1: slices 0, 1
#pragma unroll
                    for (int p = 0; p < 2; ++p) {
                        X[p] = lds128(st + 0 * BOX + p * 512);
                        LA[p] = lds128(st + 1 * BOX + p * 512);
                        LB[p] = lds128(st + 2 * BOX + p * 512);
                        G[p] = lds128(st + 3 * BOX + p * 512);
                    }
                } else {
                    const unsigned char* st = ringp + stage * STAGE + t * 4;
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        Xr[e] = lds32(st + 0 * BOX + e * 128);
                        LAr[e] = lds32(st + 1 * BOX + e * 128);
                        LBr[e] = lds32(st + 2 * BOX + e * 128);
                        Gr[e] = lds32(st + 3 * BOX + e * 128);
                    }
                }
                release_data();
                auto xv = [&](int e) { return pass == 0 ? make_float2(bfv(X[0], e), bfv(X[1], e)) : bf2(Xr[e]); };
                auto lav = [&](int e) { return pass == 0 ? make_float2(bfv(LA[0], e), bfv(LA[1], e)) : bf2(LAr[e]); };
                auto lbv = [&](int e) { return pass == 0 ? make_float2(bfv(LB[0], e), bfv(LB[1], e)) : bf2(LBr[e]); };

                // h_A(s-1) (the state line s reads) and a_B(s) of the chunk, from sweep 1,
                // half a chunk at a time (steps 7..4 first)
                float2 hAp[8], aBs[8];
                uint32_t svh[16];
                tmem::ld_x16(tstate + 32 * q + 16, svh);
                tmem::wait_ld16(svh);
#pragma unroll
                for (int e = 4; e < 8; ++e) {
                    hAp[e] = make_float2(__uint_as_float(svh[4 * (e - 4)]), __uint_as_float(svh[4 * (e - 4) + 1]));
                    aBs[e] = make_float2(__uint_as_float(svh[4 * (e - 4) + 2]), __uint_as_float(svh[4 * (e - 4) + 3]));
                }
                uint32_t dlA[2][4], dlB[2][4];  // row pass: dlambda of rows 2t+p, 8 columns (bf16 pairs)
                float2 dlAo, dlBo;               // row pass: dlambda of the odd column of a pair
                float* ds = dslot();  // upper half chunk (steps 7..4) first
                if (ds == nullptr) {
                    ++k;  // the data and weight stages of this chunk were consumed
                    fail();
                    return false;
                }
#pragma unroll
                for (int ee = 0; ee < 8; ++ee) {
                    const int e = 7 - ee;
                    const int s = 8 * q + e;
                    if (ee == 2) tmem::ld_x16(tstate + 32 * q, svh);  // steps 3..0, in flight for two steps
                    if (ee == 4) {
                        tmem::wait_ld16(svh);
#pragma unroll
                        for (int e2 = 0; e2 < 4; ++e2) {
                            hAp[e2] = make_float2(__uint_as_float(svh[4 * e2]), __uint_as_float(svh[4 * e2 + 1]));
                            aBs[e2] = make_float2(__uint_as_float(svh[4 * e2 + 2]), __uint_as_float(svh[4 * e2 + 3]));
                        }
                        dpublish();
                        ds = dslot();
                        if (ds == nullptr) {
                            ++k;
                            fail();
                            return false;
                        }
                    }
                    Taps WA, WB;
                    wrow(e, WA, WB);
                    const float2 x = xv(e), lamA = lav(e), lamB = lbv(e), ab = aBs[e];
                    // local groups: line s+1 of A starts a group, and line s of B does,
                    // exactly when s+1 is a multiple of seg
                    if (LOCAL && ((s + 1) & a.segmask) == 0) {
                        aA = make_float2(0.f, 0.f);
                        hB = make_float2(0.f, 0.f);
                    }
                    // adjoint of A at s from s+1 (taps of line s+1)
                    {
                        float2 gaA;
                        if constexpr (pass == 0) {
                            gaA = make_float2(fma_bf(e & 1, word_of(G[0], e >> 1), kOneBf2, aA.x),
                                              fma_bf(e & 1, word_of(G[1], e >> 1), kOneBf2, aA.y));
                        } else {
                            gaA = make_float2(fma_bf_lo(Gr[e], kOneBf2, aA.x), fma_bf_hi(Gr[e], kOneBf2, aA.y));
                        }
                        aA = adjoint_ga(aA, gaA, WAn, t);
                    }
                    WAn = WA;
                    // forward of B at s from s+1 (taps of B's line at s) and B's tap values
                    float2 hL, hR, m;
                    hB = fwd_step(hB, mul2(lamB, x), WB, t, hL, hR, m);
                    // tap values E = a (h_k - m): A's line s with a_A(s), B's with a_B(s).
                    // On each direction's first line the state read is zero and so are they.
                    float* const d = ds + (e & 3) * 4 * S + 2 * t;
                    *reinterpret_cast<float2*>(d + 2 * S) = mul2(ab, sub2(hL, m));
                    *reinterpret_cast<float2*>(d + 3 * S) = mul2(ab, sub2(hR, m));
                    {
                        float2 aL, aR;
                        const float2 mA = mix(hAp[e], WA, t, aL, aR);
                        *reinterpret_cast<float2*>(d + 0 * S) = mul2(aA, sub2(aL, mA));
                        *reinterpret_cast<float2*>(d + 1 * S) = mul2(aA, sub2(aR, mA));
                    }
                    // dlambda of both directions and this pass's share of dx
                    const float2 dla = mul2(x, aA), dlb = mul2(x, ab);
                    const float2 dxs = fma2(lamB, ab, mul2(lamA, aA));
                    if constexpr (pass == 0) {
                        // rows 2t, 2t+1, column s: bf16 pairs of columns (even, odd), odd first
                        if (e & 1) {
                            dlAo = dla;
                            dlBo = dlb;
                        } else {
                            dlA[0][e >> 1] = pack_bf2(dla.x, dlAo.x);
                            dlA[1][e >> 1] = pack_bf2(dla.y, dlAo.y);
                            dlB[0][e >> 1] = pack_bf2(dlb.x, dlBo.x);
                            dlB[1][e >> 1] = pack_bf2(dlb.y, dlBo.y);
                        }
                        // dx share of column s, rows 2t, 2t+1 into the column-major scratch
                        stg64_keep(dxslot + s * S + 2 * t, dxs, keep);
                    } else {
                        // row s, columns 2t, 2t+1: complete dx, dlambda of both directions
                        const float4& c0 = dxc[0][e >> 2];
                        const float4& c1 = dxc[1][e >> 2];
                        const int i = e & 3;
                        const float2 prev = make_float2(i == 0 ? c0.x : i == 1 ? c0.y : i == 2 ? c0.z : c0.w,
                                                        i == 0 ? c1.x : i == 1 ? c1.y : i == 2 ? c1.z : c1.w);
                        const float2 dxt = add2(prev, dxs);
                        stg_cs32(a.dx + (size_t)plane * S * S + s * S + 2 * t, pack_bf2(dxt.x, dxt.y));
                        stg_cs32(dlamA + s * S + 2 * t, pack_bf2(dla.x, dla.y));
                        stg_cs32(dlamB + s * S + 2 * t, pack_bf2(dlb.x, dlb.y));
                    }
                }
                if constexpr (pass == 0) {
                    // dlambda of the chunk's 8 columns: staged [row % 2][row / 2][8 columns] and
                    // written by two tiled bulk stores
                    if (t == 0) tma::bulk_wait_read();  // the previous chunk's stores have read the stage
                    __syncwarp();
#pragma unroll
                    for (int p = 0; p < 2; ++p) {
                        *reinterpret_cast<uint4*>(dlst + t * 16 + p * 512) =
                            make_uint4(dlA[p][0], dlA[p][1], dlA[p][2], dlA[p][3]);
                        *reinterpret_cast<uint4*>(dlst + BOX + t * 16 + p * 512) =
                            make_uint4(dlB[p][0], dlB[p][1], dlB[p][2], dlB[p][3]);
                    }
                    tma::fence_proxy_async();
                    __syncwarp();
                    if (t == 0) {
                        tma::store_4d(&tm_dl, dlsa, 8 * q, 0, 0, la * BC + plane);
                        tma::store_4d(&tm_dl, dlsa + BOX, 8 * q, 0, 0, lb * BC + plane);
                        tma::bulk_commit();
                    }
                } else if (q == 4 || q == 0) {
                    // every lane has used its loads of rows 32..63 (q = 4) or 0..31 (q = 0)
                    // of the dx plane: drop those dead 128-byte lines of columns 2t, 2t+1
                    __syncwarp();
                    l2_discard128(dxslot + (2 * t) * S + 8 * q);
                    l2_discard128(dxslot + (2 * t + 1) * S + 8 * q);
                }
                dpublish();
                release_w();
            }
            __syncwarp();
            return true;
        };
        if (!run_pass(std::integral_constant<int, 0>{}) || !run_pass(std::integral_constant<int, 1>{})) break;
    }
    if (t == 0) tma::bulk_wait_all();  // the dlambda stores have read shared memory
    // this warp no longer touches the tensor memory; warp 0 frees it after all
    tmem::fence_before();
    __syncwarp();
    if (t == 0) tma::mbar_arrive(done0);
    if (warp == 0) {
        if (!tma::mbar_wait(done0, 0, 10 * tma::kTimeoutNs) && t == 0) atomicExch(a.err, 1);
        __syncwarp();
        tmem::fence_after();
        tmem::dealloc(taddr, 512);
    }
}

// ---- host side ----------------------------------------------------------------------
bool make_map_cols_b(CUtensorMap* m, const void* base, uint64_t planes) {
    EncodeTiledFn fn = encode_tiled();
    if (!fn) return false;
    const cuuint64_t dims[4] = {S, S / 2, 2, planes};
    const cuuint64_t strides[3] = {2 * S * 2, S * 2, (cuuint64_t)S * S * 2};
    const cuuint32_t box[4] = {8, S / 2, 2, 1};
    const cuuint32_t es[4] = {1, 1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_map_b(CUtensorMap* m, const void* base, uint64_t planes, uint32_t box_c, uint32_t box_r) {
    EncodeTiledFn fn = encode_tiled();
    if (!fn) return false;
    const cuuint64_t dims[3] = {S, S, planes};
    const cuuint64_t strides[2] = {S * 2, S * S * 2};
    const cuuint32_t box[3] = {box_c, box_r, 1};
    const cuuint32_t es[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool c64_bwd_eligible(const Problem& p) {
    return p.d.dtype == GSPN_BF16 && p.g.shared && p.d.dir_mask == 15u && p.g.H == S && p.g.W == S &&
           S % p.g.groups == 0 && p.g.C % 8 == 0 && p.planes <= 0x7fffffff / 4 && encode_tiled() != nullptr;
}

namespace {
size_t tab_bytes(const Problem& p) { return align_up((size_t)p.g.B * 2 * S * S * sizeof(float4), kWsAlign); }
size_t sum_bytes(const Problem& p) { return align_up((size_t)p.g.B * 2 * 4 * S * S * sizeof(float), kWsAlign); }
int bwd_grid(const Problem& p, const DeviceInfo& dev) {
    const int groups = (int)(p.planes / 8);
    return groups < dev.sm_count ? groups : dev.sm_count;
}
}  // namespace

size_t c64_bwd_workspace(const Problem& p, const DeviceInfo& dev) {
    // error word | tap table (B*2*64*64 float4) | E sums (B*2*4*64*64 fp32) |
    // per-warp dx planes (grid*8 x 64*64 fp32)
    return kWsAlign + tab_bytes(p) + sum_bytes(p) + (size_t)bwd_grid(p, dev) * NCW * S * S * sizeof(float);
}

gspn_status c64_bwd(const Problem& p, const DeviceInfo& dev, const void* x, const void* logits, const void* lam,
                    const void* dout, void* dx, void* dlogits, void* dlam, void* ws, cudaStream_t s) {
    CUtensorMap xc, lc, gc, xr, lr, gr, dl;
    const uint64_t BC = (uint64_t)p.planes;
    if (!make_map_cols_b(&xc, x, BC) || !make_map_cols_b(&lc, lam, 4 * BC) || !make_map_cols_b(&gc, dout, BC) ||
        !make_map_b(&xr, x, BC, 64, 8) || !make_map_b(&lr, lam, 4 * BC, 64, 8) || !make_map_b(&gr, dout, BC, 64, 8) ||
        !make_map_cols_b(&dl, dlam, 4 * BC))
        return GSPN_ERR_UNSUPPORTED;
    char* w = static_cast<char*>(ws);
    C64BArgs a;
    a.err = reinterpret_cast<int*>(w);
    const WaitCfg wc = wait_cfg();
    a.limit = wc.limit_ns;
    a.stall = wc.stall;
    a.btab = reinterpret_cast<const float4*>(w + kWsAlign);
    a.dsum = reinterpret_cast<float*>(w + kWsAlign + tab_bytes(p));
    a.dxh = reinterpret_cast<float*>(w + kWsAlign + tab_bytes(p) + sum_bytes(p));
    a.dx = static_cast<__nv_bfloat16*>(dx);
    a.dlam = static_cast<__nv_bfloat16*>(dlam);
    a.B = p.g.B;
    a.C = p.g.C;
    a.groups = (int)(p.planes / 8);
    a.segmask = S / p.g.groups - 1;
    const int nt = p.g.B * 2 * S * LPL;
    c64b_table_kernel<__nv_bfloat16><<<(nt + 255) / 256, 256, 0, s>>>(
        static_cast<const __nv_bfloat16*>(logits), const_cast<float4*>(a.btab), a.dsum, a.err, p.g.B);
    if (cudaGetLastError() != cudaSuccess) return GSPN_ERR_CUDA;
    const bool local = p.g.groups > 1;
    const void* fn = local ? (const void*)c64b_kernel<true> : (const void*)c64b_kernel<false>;
    cudaError_t e = ensure_smem_attr(fn, SMEM_BYTES, local ? 17 : 10);
    if (e != cudaSuccess) return GSPN_ERR_CUDA;
    const int grid = bwd_grid(p, dev);
    if (local)
        c64b_kernel<true><<<grid, THREADS, SMEM_BYTES, s>>>(xc, lc, gc, xr, lr, gr, dl, a);
    else
        c64b_kernel<false><<<grid, THREADS, SMEM_BYTES, s>>>(xc, lc, gc, xr, lr, gr, dl, a);
    if (cudaGetLastError() != cudaSuccess) return GSPN_ERR_CUDA;
    const int nl = 4 * p.g.B * S * S;
    c64b_dlogits_kernel<__nv_bfloat16><<<(nl + 255) / 256, 256, 0, s>>>(
        static_cast<const __nv_bfloat16*>(logits), a.dsum, static_cast<__nv_bfloat16*>(dlogits), p.g.B);
    return cudaGetLastError() == cudaSuccess ? GSPN_OK : GSPN_ERR_CUDA;
}

}  // namespace gspn
