// gspn_compact128.cu -- fast forward for the compact (channel-shared taps)
// four-direction scan of 128x128 bf16 planes, the 2K shape of C-GSPN
// ("Scaling Parallel Sequence Models to Vision Foundation Models": 2048 px at
// patch 16, C = 1152).
//
// Operator: "Parallel Sequence Modeling via Generalized Spatial Propagation
// Network" Key designs 1-3 (row-stochastic 3-tap line scan in four directions,
// summed; local groups) with the channel-shared taps of "GSPN-2: Efficient
// Parallel Sequence Modeling" (Justification for Channel-Agnostic
// Propagation).
//
// Design (B200).  The 64x64 kernel keeps the row pass's fp32 sum of a plane in
// shared memory; at 128x128 that sum is 64 KB per plane, too much to keep
// enough planes in flight, so the pass sums take another road:
// * One CTA per SM: 4 consumer warps (one plane each, 4 consecutive channels
//   of one batch image; 32 lanes x 4 adjacent positions of a 128-wide line)
//   and 4 producer warps (lane 0 of producer w issues consumer w's TMA loads;
//   producer 0 also streams the tap table, one 16 KB chunk of 8 scan steps
//   into a ring that all 4 consumers read).
// * The two directions of a pair (left->right with right->left, top->bottom
//   with bottom->top) advance together, one per half of a float2, with the
//   packed fp32x2 FMA; lambda*x is one mixed-precision FMA on bf16 inputs.
// * A pixel is reached twice in each pass, once by each direction of the
//   pair, at steps s and 127-s, and both times by the same lane.  The first
//   arrival is parked in tensor memory (TMEM; consumer warp w owns lane
//   quarter w and all 512 columns = 64 steps x 4 positions x 2 directions);
//   the second arrival reads it back and completes the pair's sum.
// * Row pass (left->right and right->left over columns; lane t owns rows
//   4t..4t+3): the completed row sums go to a per-warp fp32 scratch plane,
//   row-major, stored with the L2 evict-last priority as 16-byte row pieces.
// * Column pass (top->bottom and bottom->top over rows; lane t owns columns
//   4t..4t+3): the first arrival adds the row sum of its row, brought in by a
//   bulk copy of 8 scratch rows (4 KB; read once, after which its L2 lines are
//   discarded); the second arrival completes the pixel and stores it, 256
//   contiguous bytes per warp and row.
// * x / lambda chunks of 8 steps arrive by TMA: column-pass chunks as one
//   128 x 8 box, row-pass chunks (8 columns x 128 rows) through a 4-D view
//   (column, row / 4, row % 4, plane), so that row 4t+p of lane t lands at
//   p*512 + t*16 and the 16-byte reads of a warp are conflict-free.
// * Every wait is bounded (2 s); on expiry the warp records an error word,
//   drains its copies and leaves.
#include <atomic>
#include <type_traits>

#include "gspn_internal.h"
#include "gspn_lane.cuh"
#include "gspn_tma.cuh"
#include "gspn_tmem.cuh"

namespace gspn {

namespace {

using namespace lane;

// ---- kernel configuration ------------------------------------------------------------
constexpr int S = 128;                 // H = W
constexpr int LPL = 32;                // lanes per line, 4 positions each
constexpr int NCW = 4;                 // consumer warps (one plane each), one per TMEM lane quarter
constexpr int NPW = 4;                 // producer warps, one per consumer
constexpr int THREADS = (NCW + NPW) * 32;
constexpr int NST = 2;                 // x / lambda stages per consumer warp
constexpr int NWS = 3;                 // tap-table stages per CTA
constexpr int NRS = 2;                 // row-sum stages per consumer warp
constexpr int BOX = 8 * S * 2;         // one x or lambda box: 8 steps x 128 positions, bf16 (2 KB)
constexpr int STAGE = 4 * BOX;         // x_A, lambda_A, x_B, lambda_B
constexpr int RTILE = 8 * S * 4;       // 8 rows of a scratch plane (4 KB)
constexpr int RSTAGE = 2 * RTILE;      // the rows of both column directions
constexpr int WCHUNK = 8 * S * 16;     // tap table rows of 8 steps (16 KB)
constexpr int RING = 0;                               // [warp][NST] data stages
constexpr int RSR = RING + NCW * NST * STAGE;         // [warp][NRS] row-sum stages
constexpr int WRING = RSR + NCW * NRS * RSTAGE;       // [NWS] tap-table stages
constexpr int BARS = WRING + NWS * WCHUNK;
constexpr int NBAR = 2 * NCW * NST + 2 * NWS + NCW * NRS + 1;
constexpr int SMEM_BYTES = 1024 + BARS + 8 * NBAR + 16;  // + the TMEM address
constexpr int CHUNKS_PER_GROUP = 32;                     // 16 row-pass + 16 column-pass chunks
static_assert(SMEM_BYTES <= 232448, "shared memory budget");
static_assert(STAGE % 1024 == 0 && RSTAGE % 1024 == 0 && WCHUNK % 1024 == 0, "TMA destinations stay aligned");

// ---- tap table pre-kernel ---------------------------------------------------------------
// wtab[((b*2 + pass)*128 + s)*128 + p*32 + t] = (-w0_A, -w0_B, w2_A, w2_B) of line
// position j = 4t + p at scan step s.  Pass 0 pairs A = left->right (line s =
// column s) with B = right->left (column 127-s), positions = rows; pass 1 pairs
// A = top->bottom (row s) with B = bottom->top (row 127-s), positions = columns.
// Taps are normalised over the valid neighbours (w0 = 0 at j = 0, w2 = 0 at j = 127).
template <typename T>
__device__ __forceinline__ void gate128(const T* lg, int pix, int j, float* w0, float* w2) {
    const float s0 = j > 0 ? sigmoidf(load_elt(lg, pix)) : 0.f;
    const float s1 = sigmoidf(load_elt(lg, S * S + pix));
    const float s2 = j < S - 1 ? sigmoidf(load_elt(lg, 2 * S * S + pix)) : 0.f;
    const float r = 1.f / (s0 + s1 + s2);
    *w0 = s0 * r;
    *w2 = s2 * r;
}

template <typename T>
__global__ void c128_weights_kernel(const T* __restrict__ logits, float4* __restrict__ wtab, int* err, int B) {
    const int idx = blockIdx.x * blockDim.x + threadIdx.x;
    if (idx == 0) *err = 0;
    if (idx >= B * 2 * S * S) return;
    const int j = idx & (S - 1), s = (idx >> 7) & (S - 1), pass = (idx >> 14) & 1, b = idx >> 15;
    const int slotA = pass ? 0 : 2, slotB = pass ? 1 : 3;
    const int pixA = pass ? s * S + j : j * S + s;
    const int pixB = pass ? (S - 1 - s) * S + j : j * S + (S - 1 - s);
    float w0a, w2a, w0b, w2b;
    gate128(logits + (size_t)(slotA * B + b) * 3 * S * S, pixA, j, &w0a, &w2a);
    gate128(logits + (size_t)(slotB * B + b) * 3 * S * S, pixB, j, &w0b, &w2b);
    const int t = j >> 2, p = j & 3;
    wtab[((size_t)(b * 2 + pass) * S + s) * S + p * LPL + t] = make_float4(-w0a, -w0b, w2a, w2b);
}

// One scan step of one lane: positions 4t..4t+3, both directions of the pair
// packed in float2.  base[p] = h[p] + lambda x, w[p] = (-w0_A, -w0_B, w2_A, w2_B).
// h'[p] = base[p] + w2 (h[p+1] - h[p]) - w0 (h[p] - h[p-1]), which equals
// w0 h[p-1] + w1 h[p] + w2 h[p+1] + lambda x for w1 = 1 - w0 - w2.  The two
// outer positions take the neighbour from the next lane; their in-lane terms
// are summed while the shuffles are in flight, so one FMA follows each shuffle.
// At the line ends the missing neighbour is the lane's own value (the shuffle
// does not wrap) times a zero tap.
__device__ __forceinline__ void step4(float2 (&h)[4], const float2 (&base)[4], const float4 (&w)[4]) {
    float2 hl, hr;
    hl.x = __shfl_up_sync(FULL, h[3].x, 1);
    hl.y = __shfl_up_sync(FULL, h[3].y, 1);
    hr.x = __shfl_down_sync(FULL, h[0].x, 1);
    hr.y = __shfl_down_sync(FULL, h[0].y, 1);
    const float2 nw0[4] = {make_float2(w[0].x, w[0].y), make_float2(w[1].x, w[1].y), make_float2(w[2].x, w[2].y),
                           make_float2(w[3].x, w[3].y)};
    const float2 w2[4] = {make_float2(w[0].z, w[0].w), make_float2(w[1].z, w[1].w), make_float2(w[2].z, w[2].w),
                          make_float2(w[3].z, w[3].w)};
    const float2 D1 = sub2(h[1], h[0]), D2 = sub2(h[2], h[1]), D3 = sub2(h[3], h[2]);
    // position 0: base + w2 D1 + (-w0) h0, then + w0 hl
    const float2 pre0 = __ffma2_rn(nw0[0], h[0], __ffma2_rn(w2[0], D1, base[0]));
    // position 3: base + (-w0) D3 - w2 h3, then + w2 hr
    const float2 pre3 = __ffma2_rn(w2[3], make_float2(-h[3].x, -h[3].y), __ffma2_rn(nw0[3], D3, base[3]));
    const float2 n1 = __ffma2_rn(nw0[1], D1, __ffma2_rn(w2[1], D2, base[1]));
    const float2 n2 = __ffma2_rn(nw0[2], D2, __ffma2_rn(w2[2], D3, base[2]));
    h[1] = n1;
    h[2] = n2;
    h[0] = __ffma2_rn(make_float2(-nw0[0].x, -nw0[0].y), hl, pre0);
    h[3] = __ffma2_rn(w2[3], hr, pre3);
}

__device__ __forceinline__ float f4(const float4& v, int i) { return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w; }
__device__ __forceinline__ void set4(float4& v, int i, float x) {
    if (i == 0) v.x = x;
    else if (i == 1) v.y = x;
    else if (i == 2) v.z = x;
    else v.w = x;
}
__device__ __forceinline__ uint2 lds64u(const unsigned char* p) { return *reinterpret_cast<const uint2*>(p); }
// order this thread's generic-proxy accesses (global and shared) before later async-proxy ones
__device__ __forceinline__ void fence_proxy_async_all() { asm volatile("fence.proxy.async;" ::: "memory"); }

struct C128Args {
    const float4* wtab;
    float* rsum;  // per consumer warp of the grid: one 128x128 fp32 scratch plane
    __nv_bfloat16* out;
    int* err;
    int B, C, segmask;
    int groups;  // B * C / 4 groups of 4 consecutive planes (one batch image each)
    uint64_t limit;  // bound of every wait on data, a stage or another warp (ns)
    int stall;       // test hook: consumer warp 0 of CTA 0 first waits on a barrier nothing completes
};

template <bool LOCAL>
__global__ void __launch_bounds__(THREADS, 1)
    c128_fwd_kernel(const __grid_constant__ CUtensorMap tm_xc, const __grid_constant__ CUtensorMap tm_lc,
                    const __grid_constant__ CUtensorMap tm_xr, const __grid_constant__ CUtensorMap tm_lr,
                    const C128Args a) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char* const smem = smem_raw + ((1024u - (tma::smem_u32(smem_raw) & 1023u)) & 1023u);
    const uint32_t sbase = tma::smem_u32(smem);
    const int warp = threadIdx.x >> 5, t = threadIdx.x & 31;
    const uint32_t xfull0 = sbase + BARS;             // [warp][stage] "data landed"
    const uint32_t xempty0 = xfull0 + 8 * NCW * NST;  // [warp][stage] "data read" (one arrival per lane)
    const uint32_t wfull0 = xempty0 + 8 * NCW * NST;  // [stage] "tap chunk landed"
    const uint32_t wempty0 = wfull0 + 8 * NWS;        // [stage] "tap chunk read" (every consumer lane)
    const uint32_t rfull0 = wempty0 + 8 * NWS;        // [warp][stage] "row sums landed"
    const uint32_t done0 = rfull0 + 8 * NCW * NRS;    // every consumer is done with the tensor memory
    uint32_t* const tslot = reinterpret_cast<uint32_t*>(smem + BARS + 8 * NBAR);
    if ((int)blockIdx.x >= a.groups) return;

    if (threadIdx.x == 0) {
        for (int i = 0; i < NCW * NST; ++i) {
            tma::mbar_init(xfull0 + 8 * i, 1);
            tma::mbar_init(xempty0 + 8 * i, 32);
        }
        for (int i = 0; i < NWS; ++i) {
            tma::mbar_init(wfull0 + 8 * i, 1);
            tma::mbar_init(wempty0 + 8 * i, NCW * 32);
        }
        for (int i = 0; i < NCW * NRS; ++i) tma::mbar_init(rfull0 + 8 * i, 1);
        tma::mbar_init(done0, NCW);
        tma::fence_barrier_init();
    }
    if (warp == 0) {  // consumer warp 0 owns the CTA's tensor memory: all 512 columns
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

    // ---------------- producer warps ----------------
    // Lane 0 of producer warp w streams consumer w's x / lambda chunks: chunk kk
    // (group blockIdx.x + (kk/32)*gridDim.x, plane 4*group + w; kk%32 = 0..15 row
    // pass, 16..31 column pass) goes to stage kk % NST once the consumer has read
    // what the stage held.  Producer 0 also streams the tap-table chunks.
    if (warp >= NCW) {
        if (t == 0) {
            const int pw = warp - NCW;
            if (pw == 0) {
                tma::prefetch_map(&tm_xc);
                tma::prefetch_map(&tm_lc);
                tma::prefetch_map(&tm_xr);
                tma::prefetch_map(&tm_lr);
            }
            bool ok = true;
            for (int kk = 0; ok && kk < nchunks; ++kk) {
                const int group = (int)blockIdx.x + (kk / CHUNKS_PER_GROUP) * (int)gridDim.x;
                const int local = kk % CHUNKS_PER_GROUP, pass = local >> 4, q = local & 15;
                if (pw == 0) {
                    const int ws = kk % NWS;
                    if (!tma::mbar_wait_sleep(wempty0 + 8 * ws, ((kk / NWS) & 1) ^ 1, 32, a.limit)) {
                        ok = false;
                        break;
                    }
                    const int b = (NCW * group) / a.C;
                    const float4* src = a.wtab + ((size_t)(b * 2 + pass) * S + 8 * q) * S;
                    tma::mbar_expect_tx(wfull0 + 8 * ws, WCHUNK);
                    tma::load_1d(sbase + WRING + ws * WCHUNK, src, WCHUNK, wfull0 + 8 * ws);
                }
                const int st = kk % NST;
                if (!tma::mbar_wait_sleep(xempty0 + 8 * (pw * NST + st), ((kk / NST) & 1) ^ 1, 32, a.limit)) {
                    ok = false;
                    break;
                }
                const int plane = NCW * group + pw;
                const uint32_t dst = sbase + RING + (pw * NST + st) * STAGE, bar = xfull0 + 8 * (pw * NST + st);
                tma::mbar_expect_tx(bar, STAGE);
                if (pass == 0) {
                    // x and lambda(left->right) at columns 8q.., x and lambda(right->left)
                    // at columns 120-8q..; all 128 rows through the (column, row/4, row%4) view
                    tma::load_4d(dst + 0 * BOX, &tm_xc, 8 * q, 0, 0, plane, bar);
                    tma::load_4d(dst + 1 * BOX, &tm_lc, 8 * q, 0, 0, 2 * BC + plane, bar);
                    tma::load_4d(dst + 2 * BOX, &tm_xc, S - 8 - 8 * q, 0, 0, plane, bar);
                    tma::load_4d(dst + 3 * BOX, &tm_lc, S - 8 - 8 * q, 0, 0, 3 * BC + plane, bar);
                } else {
                    // x and lambda(top->bottom) at rows 8q.., x and lambda(bottom->top) at rows 120-8q..
                    tma::load_3d(dst + 0 * BOX, &tm_xr, 0, 8 * q, plane, bar);
                    tma::load_3d(dst + 1 * BOX, &tm_lr, 0, 8 * q, 0 * BC + plane, bar);
                    tma::load_3d(dst + 2 * BOX, &tm_xr, 0, S - 8 - 8 * q, plane, bar);
                    tma::load_3d(dst + 3 * BOX, &tm_lr, 0, S - 8 - 8 * q, 1 * BC + plane, bar);
                }
            }
            if (!ok) atomicExch(a.err, 1);
        }
        return;
    }

    // ---------------- consumer warps: one plane each ----------------
    const unsigned char* const ringp = smem + RING + warp * NST * STAGE;
    const unsigned char* const rsp = smem + RSR + warp * NRS * RSTAGE;
    const uint32_t rsa = sbase + RSR + warp * NRS * RSTAGE;
    const unsigned char* const wring = smem + WRING;
    const uint32_t bar0 = xfull0 + 8 * NST * warp, ebar0 = xempty0 + 8 * NST * warp;
    const uint32_t rbar0 = rfull0 + 8 * NRS * warp;
    const uint32_t tq = taddr + ((uint32_t)(32 * warp) << 16);  // TMEM lane quarter of this warp
    float* const rs_plane = a.rsum + ((size_t)blockIdx.x * NCW + warp) * S * S;
    const uint64_t keep = l2_evict_last_policy();

    int k = 0;           // next chunk to consume (the same sequence for data and taps)
    int stage = 0;       // k % NST
    uint32_t phase = 0;  // bit s: parity of the next completion of data stage s
    int rs_issued = 0, rs_done = 0;  // row-sum copies of the current plane
    float2 h[4];
    __nv_bfloat16* outp = nullptr;

    auto fail = [&]() {
        if (t == 0) atomicExch(a.err, 1);
        tmem::wait_st();  // no TMEM access outlives the warp
        tmem::wait_ld_all();
        for (int kk = k; kk < k + NST && kk < nchunks; ++kk)
            tma::mbar_wait(bar0 + 8 * (kk % NST), (kk / NST) & 1, 100000000ull);
        for (int kk = k; kk < k + NWS && kk < nchunks; ++kk)
            tma::mbar_wait(wfull0 + 8 * (kk % NWS), (kk / NWS) & 1, 100000000ull);
        for (int i = rs_done; i < rs_issued; ++i)
            tma::mbar_wait(rbar0 + 8 * (i % NRS), (i / NRS) & 1, 100000000ull);
    };
    auto taps_in = [&](int kc) -> bool {
        const bool ok = tma::mbar_wait(wfull0 + 8 * (kc % NWS), (kc / NWS) & 1, a.limit);
        return __all_sync(FULL, ok);
    };
    // Stages are handed back by every lane: its generic-proxy reads of the stage
    // are ordered before the async-proxy (TMA) refill by a proxy fence, then its
    // arrival releases the stage.  Without the fence a refill was seen to land
    // before all reads of the stage had been performed.
    auto taps_out = [&](int kc) {
        tma::fence_proxy_async();
        tma::mbar_arrive(wempty0 + 8 * (kc % NWS));
    };
    auto acquire = [&]() -> bool {
        const bool ok = tma::mbar_wait(bar0 + 8 * stage, (phase >> stage) & 1u, a.limit);
        return __all_sync(FULL, ok);
    };
    // the stage is in registers: hand it back to its producer
    auto release = [&]() {
        tma::fence_proxy_async();
        tma::mbar_arrive(ebar0 + 8 * stage);
        phase ^= 1u << stage;
        ++k;
        stage = stage == NST - 1 ? 0 : stage + 1;
    };
    // row sums of column chunk i: rows 8i..8i+7 (top->bottom) and 120-8i..127-8i
    // (bottom->top) of the scratch plane, one 4 KB bulk copy each.  The caller has
    // ordered every lane's earlier accesses of the stage (and, for the first two
    // copies of a plane, its row-sum stores) before the async proxy.
    auto issue_rs = [&](int i) {
        if (t == 0) {
            const uint32_t bar = rbar0 + 8 * (i % NRS), dst = rsa + (i % NRS) * RSTAGE;
            tma::mbar_expect_tx(bar, RSTAGE);
            tma::load_1d(dst, rs_plane + 8 * i * S, RTILE, bar);
            tma::load_1d(dst + RTILE, rs_plane + (S - 8 - 8 * i) * S, RTILE, bar);
        }
        ++rs_issued;
    };
    auto tap_row = [&](const unsigned char* wc, int e, float4 (&w)[4]) {
#pragma unroll
        for (int p = 0; p < 4; ++p) w[p] = lds128f(wc + e * (S * 16) + p * (LPL * 16));
    };

    // Row pass chunk q (steps s = 8q..8q+7): left->right at column s (A), right->left
    // at column 127-s (B); lane t owns rows 4t..4t+3.  Chunks 0..7 park their values
    // (first arrivals) in TMEM; chunks 8..15 add the first arrival of the other
    // direction (step 127-s) and store the completed row sums.
    auto row_chunk = [&](int q) -> bool {
        const int kc = k;
        if (!taps_in(kc) || !acquire()) return false;
        const unsigned char* st = ringp + stage * STAGE + t * 16;
        uint4 XA[4], LA[4], XB[4], LB[4];
#pragma unroll
        for (int p = 0; p < 4; ++p) {
            XA[p] = lds128(st + 0 * BOX + p * 512);
            LA[p] = lds128(st + 1 * BOX + p * 512);
            XB[p] = lds128(st + 2 * BOX + p * 512);
            LB[p] = lds128(st + 3 * BOX + p * 512);
        }
        release();
        const unsigned char* wc = wring + (kc % NWS) * WCHUNK + t * 16;
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            // TMEM values of a half chunk: [step ee][position p][direction]
            uint32_t tv[32];
            if (q >= 8) {
                tmem::ld_x32(tq + 32 * (2 * (15 - q) + 1 - hh), tv);
                tmem::wait_ld(tv);
            }
            float4 oa[4], ob[4];  // completed row sums, 4 ascending columns per row
#pragma unroll
            for (int ee = 0; ee < 4; ++ee) {
                const int e = 4 * hh + ee;
                if (LOCAL && ((8 * q + e) & a.segmask) == 0) h[0] = h[1] = h[2] = h[3] = make_float2(0.f, 0.f);
                float4 w[4];
                tap_row(wc, e, w);
                // A reads column 8q+e = element e of its box; B column 127-8q-e = element 7-e
                float2 base[4];
#pragma unroll
                for (int p = 0; p < 4; ++p) {
                    base[p].x = fma_bf(e & 1, word_of(LA[p], e >> 1), word_of(XA[p], e >> 1), h[p].x);
                    base[p].y = fma_bf((7 - e) & 1, word_of(LB[p], (7 - e) >> 1), word_of(XB[p], (7 - e) >> 1),
                                       h[p].y);
                }
                step4(h, base, w);
                if (q < 8) {
#pragma unroll
                    for (int p = 0; p < 4; ++p) {
                        tv[ee * 8 + p * 2] = __float_as_uint(h[p].x);
                        tv[ee * 8 + p * 2 + 1] = __float_as_uint(h[p].y);
                    }
                } else {
                    // A at column s meets B's first arrival there (B's step 127-s =
                    // element 3-ee of the loaded half chunk); B at column 127-s meets A's
#pragma unroll
                    for (int p = 0; p < 4; ++p) {
                        set4(oa[p], ee, h[p].x + __uint_as_float(tv[(3 - ee) * 8 + p * 2 + 1]));
                        set4(ob[p], 3 - ee, h[p].y + __uint_as_float(tv[(3 - ee) * 8 + p * 2]));
                    }
                }
            }
            if (q < 8) {
                tmem::st_x32(tq + 32 * (2 * q + hh), tv);
            } else {
                // A covered columns 8q+4hh..+3, B columns 124-8q-4hh..+3
#pragma unroll
                for (int p = 0; p < 4; ++p) {
                    float* row = rs_plane + (4 * t + p) * S;
                    stg128_keep(row + 8 * q + 4 * hh, oa[p], keep);
                    stg128_keep(row + (S - 4) - 8 * q - 4 * hh, ob[p], keep);
                }
            }
        }
        taps_out(kc);
        return true;
    };

    // Column pass chunk q (steps s = 8q..8q+7): top->bottom at row s (A),
    // bottom->top at row 127-s (B); lane t owns columns 4t..4t+3.  Chunks 0..7 add
    // the row sums of their rows and park the values in TMEM; chunks 8..15 add the
    // first arrival of the other direction and store the finished pixels.
    auto col_chunk = [&](int q) -> bool {
        const int kc = k;
        if (!taps_in(kc) || !acquire()) return false;
        const unsigned char* st = ringp + stage * STAGE + t * 8;
        uint2 XA[8], LA[8], XB[8], LB[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            XA[e] = lds64u(st + 0 * BOX + e * 256);
            LA[e] = lds64u(st + 1 * BOX + e * 256);
            XB[e] = lds64u(st + 2 * BOX + (7 - e) * 256);  // row 127-8q-e
            LB[e] = lds64u(st + 3 * BOX + (7 - e) * 256);
        }
        release();
        const unsigned char* rs = nullptr;
        if (q < 8) {
            if (!__all_sync(FULL, tma::mbar_wait(rbar0 + 8 * (q % NRS), (q / NRS) & 1, a.limit))) return false;
            ++rs_done;
            rs = rsp + (q % NRS) * RSTAGE + t * 16;
        }
        const unsigned char* wc = wring + (kc % NWS) * WCHUNK + t * 16;
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            uint32_t tv[32];
            if (q >= 8) {
                tmem::ld_x32(tq + 32 * (2 * (15 - q) + 1 - hh), tv);
                tmem::wait_ld(tv);
            }
#pragma unroll
            for (int ee = 0; ee < 4; ++ee) {
                const int e = 4 * hh + ee, s = 8 * q + e;
                if (LOCAL && (s & a.segmask) == 0) h[0] = h[1] = h[2] = h[3] = make_float2(0.f, 0.f);
                float4 w[4];
                tap_row(wc, e, w);
                float2 base[4];
#pragma unroll
                for (int p = 0; p < 4; ++p) {
                    const uint32_t la = (p >> 1) ? LA[e].y : LA[e].x, xa = (p >> 1) ? XA[e].y : XA[e].x;
                    const uint32_t lb = (p >> 1) ? LB[e].y : LB[e].x, xb = (p >> 1) ? XB[e].y : XB[e].x;
                    base[p].x = fma_bf(p & 1, la, xa, h[p].x);
                    base[p].y = fma_bf(p & 1, lb, xb, h[p].y);
                }
                step4(h, base, w);
                if (q < 8) {
                    const float4 ra = lds128f(rs + e * 512);                // row s, columns 4t..4t+3
                    const float4 rb = lds128f(rs + RTILE + (7 - e) * 512);  // row 127-s
#pragma unroll
                    for (int p = 0; p < 4; ++p) {
                        tv[ee * 8 + p * 2] = __float_as_uint(h[p].x + f4(ra, p));
                        tv[ee * 8 + p * 2 + 1] = __float_as_uint(h[p].y + f4(rb, p));
                    }
                } else {
                    // A at row s meets B's first arrival there; B at row 127-s meets A's
                    float vA[4], vB[4];
#pragma unroll
                    for (int p = 0; p < 4; ++p) {
                        vA[p] = h[p].x + __uint_as_float(tv[(3 - ee) * 8 + p * 2 + 1]);
                        vB[p] = h[p].y + __uint_as_float(tv[(3 - ee) * 8 + p * 2]);
                    }
                    __stcs(reinterpret_cast<uint2*>(outp + s * S),
                           make_uint2(pack_bf2(vA[0], vA[1]), pack_bf2(vA[2], vA[3])));
                    __stcs(reinterpret_cast<uint2*>(outp + (S - 1 - s) * S),
                           make_uint2(pack_bf2(vB[0], vB[1]), pack_bf2(vB[2], vB[3])));
                }
            }
            if (q < 8) tmem::st_x32(tq + 32 * (2 * q + hh), tv);
        }
        if (q < 8) {
            // every lane has read the chunk's row sums: drop their 64 L2 lines (read
            // once, never written back) and refill the stage
            fence_proxy_async_all();
            __syncwarp();
            l2_discard128(rs_plane + 8 * q * S + 32 * t);
            l2_discard128(rs_plane + (S - 8 - 8 * q) * S + 32 * t);
            if (q + NRS < 8) issue_rs(q + NRS);
        }
        taps_out(kc);
        return true;
    };

    bool ok = true;
    if (a.stall && blockIdx.x == 0 && warp == 0) {
        // test hook: phase 0 of done0 needs this warp's own final arrival, so
        // this wait can only run out; the kernel then takes its error path
        ok = __all_sync(FULL, tma::mbar_wait(done0, 0, a.limit));
    }
    for (int group = blockIdx.x; ok && group < a.groups; group += gridDim.x) {
        const int plane = NCW * group + warp;
        outp = a.out + (size_t)plane * S * S + 4 * t;
        h[0] = h[1] = h[2] = h[3] = make_float2(0.f, 0.f);
        for (int q = 0; ok && q < 16; ++q) {
            if (q == 8) tmem::wait_st();  // the second half reads what the first half parked
            ok = row_chunk(q);
        }
        if (!ok) break;
        // the row sums this warp stored are read next by bulk copies (async proxy),
        // which also overwrite the row-sum stages the previous plane read
        fence_proxy_async_all();
        __syncwarp();
        rs_issued = rs_done = 0;
        for (int i = 0; i < NRS; ++i) issue_rs(i);
        h[0] = h[1] = h[2] = h[3] = make_float2(0.f, 0.f);
        for (int q = 0; ok && q < 16; ++q) {
            if (q == 8) tmem::wait_st();
            ok = col_chunk(q);
        }
    }
    if (!ok) fail();
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
// plane), one box = 8 columns of all 128 rows, laid out [row % 4][row / 4][8 columns].
bool make_map_cols(CUtensorMap* m, const void* base, uint64_t planes) {
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

// Column-pass view: (column, row, plane), one box = all 128 columns of 8 rows.
bool make_map_rows(CUtensorMap* m, const void* base, uint64_t planes) {
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

int c128_grid(const Problem& p, const DeviceInfo& dev) {
    const int groups = (int)(p.planes / NCW);
    return groups < dev.sm_count ? groups : dev.sm_count;
}
size_t c128_tab_bytes(const Problem& p) { return align_up((size_t)p.g.B * 2 * S * S * sizeof(float4), kWsAlign); }

}  // namespace

bool c128_eligible(const Problem& p) {
    return p.d.dtype == GSPN_BF16 && p.g.shared && p.d.dir_mask == 15u && p.g.H == S && p.g.W == S &&
           S % p.g.groups == 0 && p.g.C % NCW == 0 && p.planes <= 0x7fffffff / 4 && encode_tiled() != nullptr;
}

size_t c128_fwd_workspace(const Problem& p, const DeviceInfo& dev) {
    // error word | tap table (B*2*128*128 float4) | per consumer warp of the grid: a
    // 128x128 fp32 row-sum plane
    return kWsAlign + c128_tab_bytes(p) + (size_t)c128_grid(p, dev) * NCW * S * S * sizeof(float);
}

gspn_status c128_fwd(const Problem& p, const DeviceInfo& dev, const void* x, const void* logits, const void* lam,
                     void* out, void* ws, cudaStream_t s) {
    CUtensorMap xc, lc, xr, lr;
    const uint64_t BC = (uint64_t)p.planes;
    if (!make_map_cols(&xc, x, BC) || !make_map_cols(&lc, lam, 4 * BC) || !make_map_rows(&xr, x, BC) ||
        !make_map_rows(&lr, lam, 4 * BC))
        return GSPN_ERR_UNSUPPORTED;
    char* w = static_cast<char*>(ws);
    C128Args a;
    a.err = reinterpret_cast<int*>(w);
    const WaitCfg wc = wait_cfg();
    a.limit = wc.limit_ns;
    a.stall = wc.stall;
    a.wtab = reinterpret_cast<const float4*>(w + kWsAlign);
    a.rsum = reinterpret_cast<float*>(w + kWsAlign + c128_tab_bytes(p));
    a.out = static_cast<__nv_bfloat16*>(out);
    a.B = p.g.B;
    a.C = p.g.C;
    a.segmask = S / p.g.groups - 1;
    a.groups = (int)(p.planes / NCW);
    const int nw = p.g.B * 2 * S * S;
    c128_weights_kernel<__nv_bfloat16><<<(nw + 255) / 256, 256, 0, s>>>(
        static_cast<const __nv_bfloat16*>(logits), const_cast<float4*>(a.wtab), a.err, p.g.B);
    if (cudaGetLastError() != cudaSuccess) return GSPN_ERR_CUDA;
    const bool local = p.g.groups > 1;
    const void* fn = local ? (const void*)c128_fwd_kernel<true> : (const void*)c128_fwd_kernel<false>;
    if (ensure_smem_attr(fn, SMEM_BYTES, local ? 19 : 18) != cudaSuccess) return GSPN_ERR_CUDA;
    const int grid = c128_grid(p, dev);
    if (local)
        c128_fwd_kernel<true><<<grid, THREADS, SMEM_BYTES, s>>>(xc, lc, xr, lr, a);
    else
        c128_fwd_kernel<false><<<grid, THREADS, SMEM_BYTES, s>>>(xc, lc, xr, lr, a);
    return cudaGetLastError() == cudaSuccess ? GSPN_OK : GSPN_ERR_CUDA;
}

}  // namespace gspn
