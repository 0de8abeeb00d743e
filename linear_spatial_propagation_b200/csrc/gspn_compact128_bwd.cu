// gspn_compact128_bwd.cu -- fast backward for the compact (channel-shared
// taps) four-direction global or local scan of 128x128 bf16 planes, the 2K
// shape of C-GSPN ("Scaling Parallel Sequence Models to Vision Foundation
// Models": 2048 px at patch 16, C = 1152).
//
// The gradient of the line scan ("Parallel Sequence Modeling via Generalized
// Spatial Propagation Network", Key designs 1-2) is its adjoint run from the
// last line to the first ("GSPN-2: Efficient Parallel Sequence Modeling",
// Backward Benchmark).  The arithmetic is that of gspn_compact64_bwd.cu:
//   a_i[j]  = G_i[j] + a_{i+1}[j] - p0[j] - p2[j] + p0[j+1] + p2[j-1],
//             p0 = w0 a_{i+1}, p2 = w2 a_{i+1} (taps of line i+1),
//   dlambda = x a,   dx += lambda a,
//   E_0 = sum_c a (h_{i-1}[j-1] - m),  E_2 = sum_c a (h_{i-1}[j+1] - m),
//             m = the neighbour mix of h_{i-1} that line i reads,
// and dlogits from E_0, E_2 (chain rule through sigmoid and normalisation).
//
// Design (B200), per plane and per pass (row pass: A = left->right, B =
// right->left over columns s; column pass: A = top->bottom, B = bottom->top
// over rows s):
// * Sweep 1, s ascending: h_A forward and a_B adjoint.  h_A(s-1) of every
//   line goes to tensor memory (TMEM: 128 lines x 4 positions = all 512
//   columns of the warp's lane quarter); a_B(s) goes to a per-warp fp32
//   scratch plane [s][j] in L2 (evict-last).  At 64x64 both fit in TMEM; at
//   128x128 one of them has to leave the SM.
// * Sweep 2, s descending: a_A adjoint and h_B forward.  The chunk's h_A
//   states come back from TMEM, its a_B lines by one 4 KB bulk copy (read
//   once, then the L2 lines are discarded).  At every line s all four of
//   h_A(s-1), a_A(s), h_B(s+1), a_B(s) are at hand: dlambda of both
//   directions, the pass's share of dx and the tap values of both directions.
// * dx: the row pass's share goes to a second per-warp scratch plane
//   (column-major); the column pass adds its share and stores dx once.
// * Tap values: each of the 4 compute warps (4 channels of one image) stores
//   a half chunk (4 lines) of values into its shared slot; a reducer warp
//   sums the 4 slots and adds them to L2-resident fp32 sums with bulk
//   reduce-adds; two slot sets, one reducer each.  A last kernel turns the
//   sums into dlogits.
// * 4 positions per lane; lane values are float2 pairs of adjacent
//   positions, updated with the packed fp32x2 FMA.
// * x, lambda and dout chunks arrive by TMA (compute warps issue their own);
//   row-pass chunks through a 4-D view (column, row/4, row%4, plane) so that
//   row 4t+p of lane t sits at p*512 + t*16; the tap table (both directions of
//   a line in one 2 KB row) is streamed by a producer warp into a ring.
// * Every lane orders its reads of a stage before the stage's TMA refill
//   with its own proxy fence.  Every wait is bounded (2 s); on expiry the warp
//   records an error word, drains its copies and returns.
#include <atomic>
#include <type_traits>

#include "gspn_internal.h"
#include "gspn_lane.cuh"
#include "gspn_tma.cuh"
#include "gspn_tmem.cuh"

namespace gspn {

namespace {

using namespace lane;

constexpr int S = 128;
constexpr int LPL = 32;          // lanes per line, 4 positions each
constexpr int NCW = 4;           // compute warps (one plane each), one per TMEM lane quarter
constexpr int NSET = 2;          // tap-value slot sets, one reducer warp each
constexpr int THREADS = (NCW + 1 + NSET) * 32;
constexpr int NST = 2;           // data stages per compute warp
constexpr int NWS = 2;           // tap-table stages per CTA
constexpr int NAS = 2;           // a_B stages per compute warp
constexpr int BOX = 8 * S * 2;   // one tensor of a chunk: 8 lines x 128 positions, bf16 (2 KB)
constexpr int STAGE = 4 * BOX;   // x, lambda_A, lambda_B (sweep 2), dout
constexpr int ABOX = 8 * S * 4;  // a_B of 8 lines, fp32 (4 KB)
constexpr int WCHUNK = 8 * S * 16;         // tap table rows of 8 lines (16 KB)
constexpr int DSLOT = 4 * 4 * S * 4;       // one warp's tap values of a half chunk: [line][value][j] (8 KB)
constexpr int RING = 0;                                  // [warp][NST] data stages
constexpr int ARING = RING + NCW * NST * STAGE;          // [warp][NAS] a_B stages
constexpr int WRING = ARING + NCW * NAS * ABOX;          // [NWS] tap stages
constexpr int DSTG = WRING + NWS * WCHUNK;               // [set][warp] slots
constexpr int DOUT = DSTG + NSET * NCW * DSLOT;          // [set] reduced half chunk: [value][line][j]
constexpr int DLS = DOUT + NSET * DSLOT;                 // [warp] row-pass dlambda of a chunk, A then B
constexpr int BARS = DLS + NCW * 2 * BOX;
constexpr int NBAR = NCW * NST + NCW * NAS + 2 * NWS + 2 * NSET + 1;
constexpr int SMEM_BYTES = 1024 + BARS + 8 * NBAR + 16;  // + the TMEM address
constexpr int CHUNKS_PER_GROUP = 64;  // row pass sweeps 1, 2; column pass sweeps 1, 2 (16 chunks each)
static_assert(SMEM_BYTES <= 232448, "shared memory budget");
static_assert(STAGE % 1024 == 0 && ABOX % 1024 == 0 && WCHUNK % 1024 == 0 && DSLOT % 1024 == 0 && BOX % 1024 == 0,
              "TMA and bulk-copy buffers stay aligned");

// ---- backward tap table -------------------------------------------------------------
// Row (b, pass, s) holds the taps of both directions' lines at column (row
// pass) or row (column pass) s: float4 index k*32 + t, k = 0, 1: A taps of
// positions (4t, 4t+1) and (4t+2, 4t+3) as (w0, w0', w2, w2'); k = 2, 3: the
// same for B.  Pass 0: A = left->right (slot 2), B = right->left (slot 3), pixel
// (j, s); pass 1: A = top->bottom (slot 0), B = bottom->top (slot 1), pixel (s, j).
template <typename T>
__device__ __forceinline__ void gate_w128(const T* lg, int pix, int j, float* w0, float* w2) {
    const float s0 = j > 0 ? sigmoidf(load_elt(lg, pix)) : 0.f;
    const float s1 = sigmoidf(load_elt(lg, S * S + pix));
    const float s2 = j < S - 1 ? sigmoidf(load_elt(lg, 2 * S * S + pix)) : 0.f;
    const float r = 1.f / (s0 + s1 + s2);
    *w0 = s0 * r;
    *w2 = s2 * r;
}

template <typename T>
__global__ void c128b_table_kernel(const T* __restrict__ logits, float4* __restrict__ btab, float* __restrict__ dsum,
                                   int* err, int B) {
    const int idx = blockIdx.x * blockDim.x + threadIdx.x;
    if (idx == 0) *err = 0;
    const int n = B * 2 * S * LPL * 2;  // one thread per (b, pass, s, lane, position pair)
    // the tap sums start at zero: 2 directions x 2 values per pixel of each pass
    for (int q = idx; q < B * 2 * 4 * S * S; q += gridDim.x * blockDim.x) dsum[q] = 0.f;
    if (idx >= n) return;
    const int pr = idx & 1, t = (idx >> 1) & 31, s = (idx >> 6) & (S - 1), pass = (idx >> 13) & 1, b = idx >> 14;
    const int slotA = pass ? 0 : 2, slotB = pass ? 1 : 3;
    float w[2][2][2];  // [dir][position of the pair][w0, w2]
    for (int p = 0; p < 2; ++p) {
        const int j = 4 * t + 2 * pr + p, pix = pass ? s * S + j : j * S + s;
        gate_w128(logits + (size_t)(slotA * B + b) * 3 * S * S, pix, j, &w[0][p][0], &w[0][p][1]);
        gate_w128(logits + (size_t)(slotB * B + b) * 3 * S * S, pix, j, &w[1][p][0], &w[1][p][1]);
    }
    float4* row = btab + ((size_t)(b * 2 + pass) * S + s) * (4 * LPL);
    row[pr * LPL + t] = make_float4(w[0][0][0], w[0][1][0], w[0][0][1], w[0][1][1]);
    row[(2 + pr) * LPL + t] = make_float4(w[1][0][0], w[1][1][0], w[1][0][1], w[1][1][1]);
}

// dlogits from the channel sums (chain rule through w_k = s_k / sum s, s_k =
// sigmoid(logit_k)): dlogit_0 = w_0 (1 - s_0) E_0, dlogit_2 = w_2 (1 - s_2) E_2,
// dlogit_1 = -(1 - s_1) (w_0 E_0 + w_2 E_2); zero on the first line of each
// direction (its taps are never used) and on invalid taps.
template <typename T>
__global__ void c128b_dlogits_kernel(const T* __restrict__ logits, const float* __restrict__ dsum,
                                     T* __restrict__ dlogits, int B) {
    const int idx = blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= 4 * B * S * S) return;
    const int pix = idx & (S * S - 1), b = (idx >> 14) % B, slot = (idx >> 14) / B;
    const int r = pix >> 7, c = pix & (S - 1);
    const int pass = slot < 2 ? 1 : 0, dir = slot & 1;  // dir 0 = A, 1 = B
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

struct C128BArgs {
    const float4* btab;
    float* dsum;  // [B][pass][dir*2 + value][s][j]: E_0, E_2 sums
    float* dxh;   // per compute warp of the grid: the row pass's share of dx, column-major
    float* abh;   // per compute warp of the grid: a_B of sweep 1, [s][j]
    __nv_bfloat16* dx;
    __nv_bfloat16* dlam;
    int* err;
    int B, C;
    int groups;   // B * C / 4
    int segmask;  // local groups: lines per group - 1 (127 = global)
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
__device__ __forceinline__ float2 add2(float2 a, float2 b) { return __fadd2_rn(a, b); }
__device__ __forceinline__ float2 mul2(float2 a, float2 b) { return __fmul2_rn(a, b); }
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }
__device__ __forceinline__ void fence_proxy_async_all() { asm volatile("fence.proxy.async;" ::: "memory"); }

// Lane t holds positions 4t..4t+3 of a line as two float2 pairs: v[0] = (4t,
// 4t+1), v[1] = (4t+2, 4t+3).  Tap weights of a line for those positions:
struct Taps4 {
    float2 w0[2], w2[2];
};

// Neighbours of a state h: hL = h shifted right by one position (h[j-1]), hR
// = h shifted left (h[j+1]).  The shuffles rotate, so lane 0 reads position
// 127 as its left neighbour and lane 31 position 0 as its right one: both
// meet a zero tap weight (w0 at j = 0, w2 at j = 127).
__device__ __forceinline__ void nbrs4(const float2 (&h)[2], int t, float2 (&hL)[2], float2 (&hR)[2]) {
    const float l = __shfl_sync(FULL, h[1].y, (t + 31) & 31);
    const float r = __shfl_sync(FULL, h[0].x, (t + 1) & 31);
    hL[0] = make_float2(l, h[0].x);
    hL[1] = make_float2(h[0].y, h[1].x);
    hR[0] = make_float2(h[0].y, h[1].x);
    hR[1] = make_float2(h[1].y, r);
}

// Forward step h' = w0 hL + w1 h + w2 hR + lx (w1 = 1 - w0 - w2); m = h' - lx
// is the neighbour mix, for the tap values; hL, hR are the old state's.
__device__ __forceinline__ void fwd4(float2 (&h)[2], const float2 (&lx)[2], const Taps4& w, int t, float2 (&hL)[2],
                                     float2 (&hR)[2], float2 (&m)[2]) {
    nbrs4(h, t, hL, hR);
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const float2 w1 = sub2(sub2(make_float2(1.f, 1.f), w.w0[i]), w.w2[i]);
        const float2 hn = fma2(w.w2[i], hR[i], fma2(w.w0[i], hL[i], fma2(w1, h[i], lx[i])));
        m[i] = sub2(hn, lx[i]);
        h[i] = hn;
    }
}

// Neighbour mix m = w0 hL + w1 h + w2 hR of a stored state h.
__device__ __forceinline__ void mix4(const float2 (&h)[2], const Taps4& w, int t, float2 (&hL)[2], float2 (&hR)[2],
                                     float2 (&m)[2]) {
    nbrs4(h, t, hL, hR);
#pragma unroll
    for (int i = 0; i < 2; ++i) m[i] = fma2(w.w0[i], sub2(hL[i], h[i]), fma2(w.w2[i], sub2(hR[i], h[i]), h[i]));
}

// Adjoint step a' = g + W^T a with w the taps of the line that reads this one:
// a'[j] = g[j] + a[j] - p0[j] - p2[j] + p0[j+1] + p2[j-1], p0 = w0 a, p2 = w2 a.
// The rotated shuffles bring w0 a of position 0 to lane 31 and w2 a of
// position 127 to lane 0, both zero.  In-lane terms are summed while the
// shuffles are in flight.
__device__ __forceinline__ void adjoint4(float2 (&a)[2], const float2 (&g)[2], const Taps4& w, int t) {
    float2 p0[2], p2[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        p0[i] = mul2(w.w0[i], a[i]);
        p2[i] = mul2(w.w2[i], a[i]);
    }
    const float p0r = __shfl_sync(FULL, p0[0].x, (t + 1) & 31);   // w0 a at position 4t+4
    const float p2l = __shfl_sync(FULL, p2[1].y, (t + 31) & 31);  // w2 a at position 4t-1
    const float2 m1 = make_float2(-1.f, -1.f);
    const float2 n0 = add2(fma2(m1, p2[0], fma2(m1, p0[0], add2(g[0], a[0]))), make_float2(p0[0].y, p0[1].x));
    const float2 n1 = add2(fma2(m1, p2[1], fma2(m1, p0[1], add2(g[1], a[1]))), make_float2(p2[0].y, p2[1].x));
    a[0] = add2(n0, make_float2(p2l, p2[0].x));
    a[1] = add2(n1, make_float2(p0[1].y, p0r));
}

template <bool LOCAL>
__global__ void __launch_bounds__(THREADS, 1)
    c128b_kernel(const __grid_constant__ CUtensorMap tm_xc, const __grid_constant__ CUtensorMap tm_lc,
                 const __grid_constant__ CUtensorMap tm_gc, const __grid_constant__ CUtensorMap tm_xr,
                 const __grid_constant__ CUtensorMap tm_lr, const __grid_constant__ CUtensorMap tm_gr,
                 const __grid_constant__ CUtensorMap tm_dl, const C128BArgs a) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char* const smem = smem_raw + ((1024u - (tma::smem_u32(smem_raw) & 1023u)) & 1023u);
    const uint32_t sbase = tma::smem_u32(smem);
    const int warp = threadIdx.x >> 5, t = threadIdx.x & 31;
    const uint32_t xfull0 = sbase + BARS;              // [warp][stage] data landed
    const uint32_t afull0 = xfull0 + 8 * NCW * NST;    // [warp][stage] a_B lines landed
    const uint32_t wfull0 = afull0 + 8 * NCW * NAS;    // [stage] tap chunk landed
    const uint32_t wempty0 = wfull0 + 8 * NWS;         // [stage] tap chunk read (every compute lane)
    const uint32_t dfull0 = wempty0 + 8 * NWS;         // [set] the compute warps' slots are written
    const uint32_t dempty0 = dfull0 + 8 * NSET;        // [set] the reducer has read the set
    const uint32_t done0 = dempty0 + 8 * NSET;         // every compute warp is done with the tensor memory
    uint32_t* const tslot = reinterpret_cast<uint32_t*>(smem + BARS + 8 * NBAR);
    if ((int)blockIdx.x >= a.groups) return;

    if (threadIdx.x == 0) {
        for (int i = 0; i < NCW * NST; ++i) tma::mbar_init(xfull0 + 8 * i, 1);
        for (int i = 0; i < NCW * NAS; ++i) tma::mbar_init(afull0 + 8 * i, 1);
        for (int i = 0; i < NWS; ++i) {
            tma::mbar_init(wfull0 + 8 * i, 1);
            tma::mbar_init(wempty0 + 8 * i, NCW * 32);
        }
        for (int i = 0; i < NSET; ++i) {
            tma::mbar_init(dfull0 + 8 * i, NCW * 32);
            tma::mbar_init(dempty0 + 8 * i, 32);
        }
        tma::mbar_init(done0, NCW);
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

    // chunk kk of the CTA sequence: pass, sweep, chunk index q of 8 lines
    auto chunk_info = [](int kk, int& pass, int& sweep, int& q) {
        const int l = kk % CHUNKS_PER_GROUP;
        pass = l >> 5;
        sweep = (l >> 4) & 1;
        q = sweep ? 15 - (l & 15) : (l & 15);
    };

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
                const int b = (NCW * group) / a.C;
                int pass, sweep, q;
                chunk_info(kc, pass, sweep, q);
                const float4* src = a.btab + ((size_t)(b * 2 + pass) * S + 8 * q) * (4 * LPL);
                tma::mbar_expect_tx(wfull0 + 8 * ws, WCHUNK);
                tma::load_1d(sbase + WRING + ws * WCHUNK, src, WCHUNK, wfull0 + 8 * ws);
            }
        }
        return;
    }

    // ---------------- reducer warps: tap values of each sweep-2 half chunk ----------------
    // Half chunk n of the CTA (pass-major within a group, q descending, the upper 4
    // lines of a chunk first) sits in slot set n % NSET, owned by reducer warp
    // n % NSET.  It sums the 4 slots into its reduced buffer, hands the set back,
    // and adds the half chunk to the image's sums (lines 8q+4h..8q+4h+3 of each
    // of the 4 [s][j] planes) by 4 bulk reduce-adds of 2 KB.
    if (warp >= NCW + 1) {
        const int rid = warp - (NCW + 1);
        const float4* const sets = reinterpret_cast<const float4*>(smem + DSTG);
        float4* const outp = reinterpret_cast<float4*>(smem + DOUT + rid * DSLOT);
        int n = 0;
        bool ok = true;
        for (int group = blockIdx.x; ok && group < a.groups; group += gridDim.x) {
            const int b = (NCW * group) / a.C;
            for (int l = 0; l < 64; ++l, ++n) {
                const int pass = l >> 5, q = 15 - ((l >> 1) & 15), h = 1 - (l & 1), set = n % NSET;
                if (set != rid) continue;
                float* const dsum = a.dsum + (size_t)(b * 2 + pass) * 4 * S * S + (8 * q + 4 * h) * S;
                if (!__all_sync(FULL, tma::mbar_wait_sleep(dfull0 + 8 * set, (n / NSET) & 1, 128, a.limit))) {
                    ok = false;
                    break;
                }
                if (t == 0) tma::bulk_wait_read();  // this reducer's previous reduces have read its buffer
                __syncwarp();
                const float4* const src = sets + set * NCW * (DSLOT / 16);
#pragma unroll 4
                for (int i = 0; i < DSLOT / 16 / 32; ++i) {
                    // float4 f = i*32 + t of a slot: line i >> 2, value i & 3, positions 4t..4t+3
                    const int f = i * 32 + t;
                    float4 acc = src[f];
#pragma unroll
                    for (int w = 1; w < NCW; ++w) {
                        const float4 v = src[w * (DSLOT / 16) + f];
                        acc.x += v.x;
                        acc.y += v.y;
                        acc.z += v.z;
                        acc.w += v.w;
                    }
                    outp[((i & 3) * 4 + (i >> 2)) * 32 + t] = acc;  // [value][line][j]
                }
                tma::mbar_arrive(dempty0 + 8 * set);  // every lane: its reads of the set are done
                tma::fence_proxy_async();             // its writes of the buffer come before the reduces
                __syncwarp();
                if (t == 0) {
                    for (int v = 0; v < 4; ++v)
                        tma::reduce_add_f32(dsum + (size_t)v * S * S, sbase + DOUT + rid * DSLOT + v * 2048, 2048);
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

    // ---------------- compute warps ----------------
    const uint32_t ring = sbase + RING + warp * NST * STAGE;
    const unsigned char* const ringp = smem + RING + warp * NST * STAGE;
    const uint32_t aring = sbase + ARING + warp * NAS * ABOX;
    const unsigned char* const aringp = smem + ARING + warp * NAS * ABOX;
    float* const dxslot = a.dxh + ((size_t)blockIdx.x * NCW + warp) * S * S;  // [column][row]
    float* const abslot = a.abh + ((size_t)blockIdx.x * NCW + warp) * S * S;  // [line][position]
    // h_A(s-1) of line s: lane t of TMEM quarter `warp`, columns 4s..4s+3
    const uint32_t tstate = taddr + ((uint32_t)(32 * warp) << 16);
    unsigned char* const dlst = smem + DLS + warp * 2 * BOX;
    const uint32_t dlsa = sbase + DLS + warp * 2 * BOX;
    const uint64_t keep = l2_evict_last_policy();
    const unsigned char* const wring = smem + WRING;
    const uint32_t bar0 = xfull0 + 8 * NST * warp;
    const uint32_t abar0 = afull0 + 8 * NAS * warp;

    if (t == 0) {
        tma::prefetch_map(&tm_xc);
        tma::prefetch_map(&tm_lc);
        tma::prefetch_map(&tm_gc);
        tma::prefetch_map(&tm_xr);
        tma::prefetch_map(&tm_lr);
        tma::prefetch_map(&tm_gr);
        tma::prefetch_map(&tm_dl);
    }

    // Data of chunk kk (lane 0): x, lambda_A, lambda_B (sweep 2 only) and dout of
    // the chunk's 8 lines: row pass [row % 4][row / 4][8 columns] through the 4-D
    // view, column pass [8 rows][128 columns].
    auto issue = [&](int kk) {
        if (kk >= nchunks) return;
        const int group = (int)blockIdx.x + (kk / CHUNKS_PER_GROUP) * (int)gridDim.x;
        const int plane = NCW * group + warp;
        int pass, sweep, q;
        chunk_info(kk, pass, sweep, q);
        const int st = kk % NST;
        const uint32_t dst = ring + st * STAGE, bar = bar0 + 8 * st;
        tma::mbar_expect_tx(bar, sweep ? 4 * BOX : 3 * BOX);
        const int la = pass ? 0 : 2, lb = pass ? 1 : 3;  // lambda slots of A and B
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
    };
    if (t == 0)
        for (int kk = 0; kk < NST; ++kk) issue(kk);

    int k = 0, stage = 0;
    uint32_t phase = 0;
    int ab_issued = 0, ab_done = 0;  // a_B copies of the current sweep 2
    auto fail = [&]() {
        if (t == 0) atomicExch(a.err, 1);
        tmem::wait_st();  // no TMEM access outlives the warp
        tmem::wait_ld_all();
        for (int kk = k; kk < k + NST && kk < nchunks; ++kk)
            tma::mbar_wait(bar0 + 8 * (kk % NST), (kk / NST) & 1, 100000000ull);
        for (int kk = k; kk < k + NWS && kk < nchunks; ++kk)
            tma::mbar_wait(wfull0 + 8 * (kk % NWS), (kk / NWS) & 1, 100000000ull);
        for (int i = ab_done; i < ab_issued; ++i)
            tma::mbar_wait(abar0 + 8 * (i % NAS), (i / NAS) & 1, 100000000ull);
        if (t == 0) tma::bulk_wait_all();
    };
    auto acquire = [&]() -> bool {
        const bool ok1 = tma::mbar_wait(bar0 + 8 * stage, (phase >> stage) & 1u, a.limit);
        const bool ok2 = tma::mbar_wait(wfull0 + 8 * (k % NWS), (k / NWS) & 1, a.limit);
        return __all_sync(FULL, ok1 && ok2);
    };
    // the data stage is in registers: refill it (every lane orders its reads of
    // the stage before the async-proxy writes with a proxy fence of its own)
    auto release_data = [&]() {
        tma::fence_proxy_async();
        __syncwarp();
        if (t == 0) issue(k + NST);
        phase ^= 1u << stage;
        stage = stage == NST - 1 ? 0 : stage + 1;
    };
    // done with the tap stage of chunk k
    auto release_w = [&]() {
        tma::fence_proxy_async();
        tma::mbar_arrive(wempty0 + 8 * (k % NWS));
        ++k;
    };
    // taps of line e of the current tap stage, both directions
    auto wrow = [&](int e, Taps4& A, Taps4& Bt) {
        const unsigned char* src = wring + (k % NWS) * WCHUNK + e * 2048 + t * 16;
        float4 v[4];
#pragma unroll
        for (int kq = 0; kq < 4; ++kq) v[kq] = lds128f(src + kq * 512);
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            A.w0[i] = make_float2(v[i].x, v[i].y);
            A.w2[i] = make_float2(v[i].z, v[i].w);
            Bt.w0[i] = make_float2(v[2 + i].x, v[2 + i].y);
            Bt.w2[i] = make_float2(v[2 + i].z, v[2 + i].w);
        }
    };
    // a_B lines of sweep-2 chunk number i (chunk q = 15 - i): one 4 KB bulk copy
    // of the scratch plane into stage i % NAS.  The caller has ordered every
    // lane's earlier accesses before the async proxy.
    auto issue_ab = [&](int i) {
        if (t == 0) {
            const uint32_t bar = abar0 + 8 * (i % NAS);
            tma::mbar_expect_tx(bar, ABOX);
            tma::load_1d(aring + (i % NAS) * ABOX, abslot + 8 * (15 - i) * S, ABOX, bar);
        }
        ++ab_issued;
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

    const Taps4 zero_taps = {{make_float2(0.f, 0.f), make_float2(0.f, 0.f)}, {make_float2(0.f, 0.f), make_float2(0.f, 0.f)}};
    bool stalled = false;
    if (a.stall && blockIdx.x == 0 && warp == 0 &&
        !__all_sync(FULL, tma::mbar_wait(done0, 0, a.limit))) {
        // test hook: phase 0 of done0 needs this warp's own final arrival, so the
        // wait above can only run out; take the error path
        fail();
        stalled = true;
    }
    for (int group = blockIdx.x; !stalled && group < a.groups; group += gridDim.x) {
        const int plane = NCW * group + warp;

        auto run_pass = [&](auto pass_c) -> bool {
            constexpr int pass = decltype(pass_c)::value;
            const int la = pass ? 0 : 2, lb = pass ? 1 : 3;
            __nv_bfloat16* const dlamA = a.dlam + ((size_t)la * BC + plane) * S * S;
            __nv_bfloat16* const dlamB = a.dlam + ((size_t)lb * BC + plane) * S * S;

            // ---------------- sweep 1: h_A forward and a_B adjoint, s ascending ----------------
            float2 hA[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
            float2 aB[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
            Taps4 WBp = zero_taps;  // B taps of line s-1 (none before s = 0: a_B(-1) = 0)
            for (int q = 0; q < 16; ++q) {
                if (!acquire()) { fail(); return false; }
                uint4 X[4] = {}, LA[4] = {}, G[4] = {};
                uint2 Xr[8] = {}, LAr[8] = {}, Gr[8] = {};
                if constexpr (pass == 0) {
                    const unsigned char* st = ringp + stage * STAGE + t * 16;  // row 4t+p at p*512
#pragma unroll
                    for (int p = 0; p < 4; ++p) {
                        X[p] = lds128(st + 0 * BOX + p * 512);
                        LA[p] = lds128(st + 1 * BOX + p * 512);
                        G[p] = lds128(st + 3 * BOX + p * 512);
                    }
                } else {
                    const unsigned char* st = ringp + stage * STAGE + t * 8;  // columns 4t..4t+3 of row e
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        Xr[e] = *reinterpret_cast<const uint2*>(st + 0 * BOX + e * 256);
                        LAr[e] = *reinterpret_cast<const uint2*>(st + 1 * BOX + e * 256);
                        Gr[e] = *reinterpret_cast<const uint2*>(st + 3 * BOX + e * 256);
                    }
                }
                release_data();
                uint32_t sv[32];  // h_A(s-1) of the chunk's 8 lines, for TMEM
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const int s = 8 * q + e;
                    Taps4 WA, WB;
                    wrow(e, WA, WB);
                    float2 x[2], lam[2], g[2];
#pragma unroll
                    for (int i = 0; i < 2; ++i) {
                        if constexpr (pass == 0) {
                            x[i] = make_float2(bfv(X[2 * i], e), bfv(X[2 * i + 1], e));
                            lam[i] = make_float2(bfv(LA[2 * i], e), bfv(LA[2 * i + 1], e));
                            g[i] = make_float2(bfv(G[2 * i], e), bfv(G[2 * i + 1], e));
                        } else {
                            x[i] = bf2(i ? Xr[e].y : Xr[e].x);
                            lam[i] = bf2(i ? LAr[e].y : LAr[e].x);
                            g[i] = bf2(i ? Gr[e].y : Gr[e].x);
                        }
                    }
                    // local groups: line s of A starts a group, and line s-1 of B (the
                    // next in B's order) starts one, exactly when s is a multiple of seg
                    if (LOCAL && (s & a.segmask) == 0) {
                        hA[0] = hA[1] = aB[0] = aB[1] = make_float2(0.f, 0.f);
                    }
                    sv[4 * e + 0] = __float_as_uint(hA[0].x);
                    sv[4 * e + 1] = __float_as_uint(hA[0].y);
                    sv[4 * e + 2] = __float_as_uint(hA[1].x);
                    sv[4 * e + 3] = __float_as_uint(hA[1].y);
                    const float2 lx[2] = {mul2(lam[0], x[0]), mul2(lam[1], x[1])};
                    float2 hL[2], hR[2], m[2];
                    fwd4(hA, lx, WA, t, hL, hR, m);
                    adjoint4(aB, g, WBp, t);
                    stg128_keep(abslot + s * S + 4 * t, make_float4(aB[0].x, aB[0].y, aB[1].x, aB[1].y), keep);
                    WBp = WB;
                }
                tmem::st_x32(tstate + 32 * q, sv);
                release_w();
            }
            tmem::wait_st();  // sweep 2 reads what sweep 1 stored
            // the a_B lines stored above (generic proxy) are read next by bulk
            // copies, which also refill the stages the previous sweep 2 read
            fence_proxy_async_all();
            __syncwarp();
            ab_issued = ab_done = 0;
            for (int i = 0; i < NAS; ++i) issue_ab(i);

            // ---------------- sweep 2: s descending ----------------
            float2 aA[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
            float2 hB[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
            Taps4 WAn = zero_taps;  // A taps of line s+1 (none after s = 127: a_A(128) = 0)
            for (int qq = 0; qq < 16; ++qq) {
                const int q = 15 - qq;
                // column pass: the row pass's dx share of columns 4t..4t+3, rows
                // 8q..8q+7 (the scratch plane is column-major)
                float4 dxc[4][2];
                if constexpr (pass == 1) {
#pragma unroll
                    for (int c = 0; c < 4; ++c)
#pragma unroll
                        for (int h = 0; h < 2; ++h) dxc[c][h] = ldg128_keep(dxslot + (4 * t + c) * S + 8 * q + 4 * h, keep);
                }
                if (!acquire()) { fail(); return false; }
                uint4 X[4] = {}, LA[4] = {}, LB[4] = {}, G[4] = {};
                uint2 Xr[8] = {}, LAr[8] = {}, LBr[8] = {}, Gr[8] = {};
                if constexpr (pass == 0) {
                    const unsigned char* st = ringp + stage * STAGE + t * 16;
#pragma unroll
                    for (int p = 0; p < 4; ++p) {
                        X[p] = lds128(st + 0 * BOX + p * 512);
                        LA[p] = lds128(st + 1 * BOX + p * 512);
                        LB[p] = lds128(st + 2 * BOX + p * 512);
                        G[p] = lds128(st + 3 * BOX + p * 512);
                    }
                } else {
                    const unsigned char* st = ringp + stage * STAGE + t * 8;
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        Xr[e] = *reinterpret_cast<const uint2*>(st + 0 * BOX + e * 256);
                        LAr[e] = *reinterpret_cast<const uint2*>(st + 1 * BOX + e * 256);
                        LBr[e] = *reinterpret_cast<const uint2*>(st + 2 * BOX + e * 256);
                        Gr[e] = *reinterpret_cast<const uint2*>(st + 3 * BOX + e * 256);
                    }
                }
                release_data();
                if (!__all_sync(FULL, tma::mbar_wait(abar0 + 8 * (qq % NAS), (qq / NAS) & 1, a.limit))) {
                    ++k;  // the data stage of this chunk was consumed
                    fail();
                    return false;
                }
                ++ab_done;
                const unsigned char* const abst = aringp + (qq % NAS) * ABOX + t * 16;  // a_B line e at e*512
                uint32_t dlA[4][4], dlB[4][4];  // row pass: dlambda of rows 4t+p, 8 columns (bf16 pairs)
                float2 dlAo[2], dlBo[2];        // row pass: dlambda of the odd column of a pair
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const int h = 1 - hh;  // the upper half chunk (lines 4..7) first
                    // h_A(s-1) of the half chunk's 4 lines
                    uint32_t hv[16];
                    tmem::ld_x16(tstate + 32 * q + 16 * h, hv);
                    tmem::wait_ld16(hv);
                    float* const ds = dslot();
                    if (ds == nullptr) {
                        ++k;  // the data stage of this chunk was consumed
                        fail();
                        return false;
                    }
#pragma unroll
                    for (int ee = 0; ee < 4; ++ee) {
                        const int e4 = 3 - ee, e = 4 * h + e4, s = 8 * q + e;
                        Taps4 WA, WB;
                        wrow(e, WA, WB);
                        float2 x[2], lamA[2], lamB[2], g[2];
#pragma unroll
                        for (int i = 0; i < 2; ++i) {
                            if constexpr (pass == 0) {
                                x[i] = make_float2(bfv(X[2 * i], e), bfv(X[2 * i + 1], e));
                                lamA[i] = make_float2(bfv(LA[2 * i], e), bfv(LA[2 * i + 1], e));
                                lamB[i] = make_float2(bfv(LB[2 * i], e), bfv(LB[2 * i + 1], e));
                                g[i] = make_float2(bfv(G[2 * i], e), bfv(G[2 * i + 1], e));
                            } else {
                                x[i] = bf2(i ? Xr[e].y : Xr[e].x);
                                lamA[i] = bf2(i ? LAr[e].y : LAr[e].x);
                                lamB[i] = bf2(i ? LBr[e].y : LBr[e].x);
                                g[i] = bf2(i ? Gr[e].y : Gr[e].x);
                            }
                        }
                        const float4 abv = lds128f(abst + e * 512);
                        const float2 ab[2] = {make_float2(abv.x, abv.y), make_float2(abv.z, abv.w)};
                        // local groups: line s+1 of A starts a group, and line s of B does,
                        // exactly when s+1 is a multiple of seg
                        if (LOCAL && ((s + 1) & a.segmask) == 0) {
                            aA[0] = aA[1] = hB[0] = hB[1] = make_float2(0.f, 0.f);
                        }
                        // adjoint of A at s from s+1 (taps of line s+1)
                        adjoint4(aA, g, WAn, t);
                        WAn = WA;
                        // forward of B at s from s+1 (taps of B's line s)
                        const float2 lxB[2] = {mul2(lamB[0], x[0]), mul2(lamB[1], x[1])};
                        float2 hL[2], hR[2], m[2];
                        fwd4(hB, lxB, WB, t, hL, hR, m);
                        // A's state at line s-1 and its neighbour mix with A's taps of line s
                        const float2 hAp[2] = {
                            make_float2(__uint_as_float(hv[4 * e4]), __uint_as_float(hv[4 * e4 + 1])),
                            make_float2(__uint_as_float(hv[4 * e4 + 2]), __uint_as_float(hv[4 * e4 + 3]))};
                        float2 aL[2], aR[2], mA[2];
                        mix4(hAp, WA, t, aL, aR, mA);
                        // tap values E = a (h_k - m); zero on each direction's first line,
                        // where the state read is zero
                        float* const d = ds + e4 * 4 * S + 4 * t;
                        float2 v[4][2];
#pragma unroll
                        for (int i = 0; i < 2; ++i) {
                            v[0][i] = mul2(aA[i], sub2(aL[i], mA[i]));
                            v[1][i] = mul2(aA[i], sub2(aR[i], mA[i]));
                            v[2][i] = mul2(ab[i], sub2(hL[i], m[i]));
                            v[3][i] = mul2(ab[i], sub2(hR[i], m[i]));
                        }
#pragma unroll
                        for (int vv = 0; vv < 4; ++vv)
                            *reinterpret_cast<float4*>(d + vv * S) = make_float4(v[vv][0].x, v[vv][0].y, v[vv][1].x, v[vv][1].y);
                        // dlambda of both directions and this pass's share of dx
                        float2 dla[2], dlb[2], dxs[2];
#pragma unroll
                        for (int i = 0; i < 2; ++i) {
                            dla[i] = mul2(x[i], aA[i]);
                            dlb[i] = mul2(x[i], ab[i]);
                            dxs[i] = fma2(lamB[i], ab[i], mul2(lamA[i], aA[i]));
                        }
                        if constexpr (pass == 0) {
                            // rows 4t..4t+3, column s: bf16 pairs of columns (even, odd), odd first
                            if (e & 1) {
                                dlAo[0] = dla[0];
                                dlAo[1] = dla[1];
                                dlBo[0] = dlb[0];
                                dlBo[1] = dlb[1];
                            } else {
#pragma unroll
                                for (int i = 0; i < 2; ++i) {
                                    dlA[2 * i][e >> 1] = pack_bf2(dla[i].x, dlAo[i].x);
                                    dlA[2 * i + 1][e >> 1] = pack_bf2(dla[i].y, dlAo[i].y);
                                    dlB[2 * i][e >> 1] = pack_bf2(dlb[i].x, dlBo[i].x);
                                    dlB[2 * i + 1][e >> 1] = pack_bf2(dlb[i].y, dlBo[i].y);
                                }
                            }
                            // dx share of column s, rows 4t..4t+3 into the column-major scratch
                            stg128_keep(dxslot + s * S + 4 * t, make_float4(dxs[0].x, dxs[0].y, dxs[1].x, dxs[1].y), keep);
                        } else {
                            // row s, columns 4t..4t+3: complete dx, dlambda of both directions
                            float f[4];
#pragma unroll
                            for (int c = 0; c < 4; ++c) {
                                const float4& src = dxc[c][e >> 2];
                                const int i = e & 3;
                                const float prev = i == 0 ? src.x : i == 1 ? src.y : i == 2 ? src.z : src.w;
                                f[c] = prev + ((c & 1) ? dxs[c >> 1].y : dxs[c >> 1].x);
                            }
                            __stcs(reinterpret_cast<uint2*>(a.dx + (size_t)plane * S * S + s * S + 4 * t),
                                   make_uint2(pack_bf2(f[0], f[1]), pack_bf2(f[2], f[3])));
                            __stcs(reinterpret_cast<uint2*>(dlamA + s * S + 4 * t),
                                   make_uint2(pack_bf2(dla[0].x, dla[0].y), pack_bf2(dla[1].x, dla[1].y)));
                            __stcs(reinterpret_cast<uint2*>(dlamB + s * S + 4 * t),
                                   make_uint2(pack_bf2(dlb[0].x, dlb[0].y), pack_bf2(dlb[1].x, dlb[1].y)));
                        }
                    }
                    dpublish();
                }
                if constexpr (pass == 0) {
                    // dlambda of the chunk's 8 columns: staged [row % 4][row / 4][8 columns]
                    // and written by two tiled bulk stores through the 4-D view
                    if (t == 0) tma::bulk_wait_read();  // the previous chunk's stores have read the stage
                    __syncwarp();
#pragma unroll
                    for (int p = 0; p < 4; ++p) {
                        *reinterpret_cast<uint4*>(dlst + p * 512 + t * 16) =
                            make_uint4(dlA[p][0], dlA[p][1], dlA[p][2], dlA[p][3]);
                        *reinterpret_cast<uint4*>(dlst + BOX + p * 512 + t * 16) =
                            make_uint4(dlB[p][0], dlB[p][1], dlB[p][2], dlB[p][3]);
                    }
                    tma::fence_proxy_async();
                    __syncwarp();
                    if (t == 0) {
                        tma::store_4d(&tm_dl, dlsa, 8 * q, 0, 0, la * BC + plane);
                        tma::store_4d(&tm_dl, dlsa + BOX, 8 * q, 0, 0, lb * BC + plane);
                        tma::bulk_commit();
                    }
                } else if ((q & 3) == 0) {
                    // rows 8q..8q+31 of columns 4t..4t+3 have been read: drop those dead
                    // 128-byte lines of the dx plane
#pragma unroll
                    for (int c = 0; c < 4; ++c) l2_discard128(dxslot + (4 * t + c) * S + 8 * q);
                }
                // the chunk's a_B lines are read: drop them from L2 and refill the stage
                fence_proxy_async_all();
                __syncwarp();
                l2_discard128(abslot + 8 * q * S + 32 * t);
                if (qq + NAS < 16) issue_ab(qq + NAS);
                release_w();
            }
            __syncwarp();
            return true;
        };
        if (!run_pass(std::integral_constant<int, 0>{}) || !run_pass(std::integral_constant<int, 1>{})) break;
    }
    if (t == 0) tma::bulk_wait_all();  // the dlambda stores have read shared memory
    // this warp no longer touches the tensor memory; warp 0 frees it after all
    tmem::wait_st();
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
// Row-pass view of a stack of 128x128 bf16 planes: (column, row / 4, row % 4,
// plane); one box = 8 columns of all 128 rows, laid out [row % 4][row / 4][8 columns].
bool make_map_cols_b(CUtensorMap* m, const void* base, uint64_t planes) {
    EncodeTiledFn fn = encode_tiled();
    if (!fn) return false;
    const cuuint64_t dims[4] = {S, S / 4, 4, planes};
    const cuuint64_t strides[3] = {4 * S * 2, S * 2, (cuuint64_t)S * S * 2};
    const cuuint32_t box[4] = {8, S / 4, 4, 1};
    const cuuint32_t es[4] = {1, 1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Column-pass view: (column, row, plane); one box = all 128 columns of 8 rows.
bool make_map_rows_b(CUtensorMap* m, const void* base, uint64_t planes) {
    EncodeTiledFn fn = encode_tiled();
    if (!fn) return false;
    const cuuint64_t dims[3] = {S, S, planes};
    const cuuint64_t strides[2] = {S * 2, (cuuint64_t)S * S * 2};
    const cuuint32_t box[3] = {S, 8, 1};
    const cuuint32_t es[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int c128b_grid(const Problem& p, const DeviceInfo& dev) {
    const int groups = (int)(p.planes / NCW);
    return groups < dev.sm_count ? groups : dev.sm_count;
}
size_t c128b_tab_bytes(const Problem& p) { return align_up((size_t)p.g.B * 2 * S * S * sizeof(float4), kWsAlign); }
size_t c128b_sum_bytes(const Problem& p) { return align_up((size_t)p.g.B * 2 * 4 * S * S * sizeof(float), kWsAlign); }

}  // namespace

bool c128_bwd_eligible(const Problem& p) {
    return p.d.dtype == GSPN_BF16 && p.g.shared && p.d.dir_mask == 15u && p.g.H == S && p.g.W == S &&
           S % p.g.groups == 0 && p.g.C % NCW == 0 && p.planes <= 0x7fffffff / 4 && encode_tiled() != nullptr;
}

size_t c128_bwd_workspace(const Problem& p, const DeviceInfo& dev) {
    // error word | tap table (B*2*128*128 float4) | E sums (B*2*4*128*128 fp32) |
    // per compute warp of the grid: a dx plane and an a_B plane (128x128 fp32 each)
    return kWsAlign + c128b_tab_bytes(p) + c128b_sum_bytes(p) +
           (size_t)c128b_grid(p, dev) * NCW * 2 * S * S * sizeof(float);
}

gspn_status c128_bwd(const Problem& p, const DeviceInfo& dev, const void* x, const void* logits, const void* lam,
                     const void* dout, void* dx, void* dlogits, void* dlam, void* ws, cudaStream_t s) {
    CUtensorMap xc, lc, gc, xr, lr, gr, dl;
    const uint64_t BC = (uint64_t)p.planes;
    if (!make_map_cols_b(&xc, x, BC) || !make_map_cols_b(&lc, lam, 4 * BC) || !make_map_cols_b(&gc, dout, BC) ||
        !make_map_rows_b(&xr, x, BC) || !make_map_rows_b(&lr, lam, 4 * BC) || !make_map_rows_b(&gr, dout, BC) ||
        !make_map_cols_b(&dl, dlam, 4 * BC))
        return GSPN_ERR_UNSUPPORTED;
    const int grid = c128b_grid(p, dev);
    char* w = static_cast<char*>(ws);
    C128BArgs a;
    a.err = reinterpret_cast<int*>(w);
    const WaitCfg wc = wait_cfg();
    a.limit = wc.limit_ns;
    a.stall = wc.stall;
    a.btab = reinterpret_cast<const float4*>(w + kWsAlign);
    a.dsum = reinterpret_cast<float*>(w + kWsAlign + c128b_tab_bytes(p));
    a.dxh = reinterpret_cast<float*>(w + kWsAlign + c128b_tab_bytes(p) + c128b_sum_bytes(p));
    a.abh = a.dxh + (size_t)grid * NCW * S * S;
    a.dx = static_cast<__nv_bfloat16*>(dx);
    a.dlam = static_cast<__nv_bfloat16*>(dlam);
    a.B = p.g.B;
    a.C = p.g.C;
    a.groups = (int)(p.planes / NCW);
    a.segmask = S / p.g.groups - 1;
    const int nt = p.g.B * 2 * S * LPL * 2;
    c128b_table_kernel<__nv_bfloat16><<<(nt + 255) / 256, 256, 0, s>>>(
        static_cast<const __nv_bfloat16*>(logits), const_cast<float4*>(a.btab), a.dsum, a.err, p.g.B);
    if (cudaGetLastError() != cudaSuccess) return GSPN_ERR_CUDA;
    const bool local = p.g.groups > 1;
    const void* fn = local ? (const void*)c128b_kernel<true> : (const void*)c128b_kernel<false>;
    if (ensure_smem_attr(fn, SMEM_BYTES, local ? 21 : 20) != cudaSuccess) return GSPN_ERR_CUDA;
    if (local)
        c128b_kernel<true><<<grid, THREADS, SMEM_BYTES, s>>>(xc, lc, gc, xr, lr, gr, dl, a);
    else
        c128b_kernel<false><<<grid, THREADS, SMEM_BYTES, s>>>(xc, lc, gc, xr, lr, gr, dl, a);
    if (cudaGetLastError() != cudaSuccess) return GSPN_ERR_CUDA;
    const int nl = 4 * p.g.B * S * S;
    c128b_dlogits_kernel<__nv_bfloat16><<<(nl + 255) / 256, 256, 0, s>>>(
        static_cast<const __nv_bfloat16*>(logits), a.dsum, static_cast<__nv_bfloat16*>(dlogits), p.g.B);
    return cudaGetLastError() == cudaSuccess ? GSPN_OK : GSPN_ERR_CUDA;
}

}  // namespace gspn
