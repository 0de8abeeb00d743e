// gspn_compact64.cu -- fast forward for the compact (channel-shared taps)
// four-direction scan of 64x64 bf16 planes, the 1K foundation shape
// (C-GSPN, "Scaling Parallel Sequence Models to Vision Foundation Models":
// batch 32, C = 1152, 1024 px at patch 16).
//
// Operator: "Parallel Sequence Modeling via Generalized Spatial Propagation
// Network" Key designs 1-3 (row-stochastic 3-tap line scan in four directions,
// summed; local groups) with the channel-shared taps of "GSPN-2: Efficient
// Parallel Sequence Modeling" (Justification for Channel-Agnostic
// Propagation: W kron I(C), per-channel lambda).
//
// Design (B200):
// * The tap weights depend only on (b, pixel, direction).  A pre-kernel turns
//   the logits into normalised (-w0, w2) pairs once per (b, pixel,
//   direction) -- w1 = 1 - w0 - w2 -- in scan order: table row b*128 + l
//   holds the 64 positions of plane step l (64 row-pass then 64 column-pass
//   steps), 1 KB per row.
// * A CTA (one per SM) scans groups of 8 consecutive planes of one batch
//   image, one plane per consumer warp, 32 lanes per 64-wide line and 2
//   positions per lane.  The 8 warps step through the same sequence of
//   8-step chunks, so each chunk's tap weights (8 table rows, 8 KB) arrive
//   once per CTA by one bulk copy into shared memory.  Four weight warps,
//   one per lane quarter of the tensor memory (TMEM), each read the chunk
//   once and write it into their quarter (lane t: the taps of positions 2t,
//   2t+1, 8 columns per step); the two consumer warps of a quarter read two
//   steps' columns with one tcgen05.ld, a pair ahead.  Shared memory thus
//   serves each chunk four times instead of eight, and the consumers issue
//   no weight loads from it.  Chunks rotate over 4 stages (64 TMEM columns
//   each); a quarter's stage is refilled once both its consumers loaded it.
// * The two directions of a pair (left->right with right->left, top->bottom
//   with bottom->top) advance together: lane values are float2 (one
//   direction per half) and the update is the packed fp32x2 FMA of sm_100;
//   lambda*x is one mixed-precision FMA with bf16 inputs.
// * Update in difference form, h'[p] = h[p] + lambda x + w2 (h[p+1] - h[p])
//   - w0 (h[p] - h[p-1]), equal to w0 h[p-1] + w1 h[p] + w2 h[p+1] + lambda x
//   for w1 = 1 - w0 - w2; the line ends have w0 = 0 / w2 = 0.  Neighbours
//   across lanes come from two shuffles per direction and step.
// * Row pass first (left->right and right->left over columns), then column
//   pass (top->bottom and bottom->top over rows).  The row pass leaves its
//   sum in an fp32 plane in shared memory (Hacc); the column pass adds its two
//   directions and writes each output row once, 128 contiguous bytes.  In
//   each pass the direction that reaches a pixel first stores, the second
//   adds, so every Hacc element is stored and loaded the fewest times.
// * x / lambda are streamed by TMA into a per-warp ring of 4 KB stages (8
//   scan steps each): column chunks (8 columns x 64 rows) for the row pass
//   and row chunks (64 columns x 8 rows) for the column pass.  A column chunk
//   is one box of a 4-D view of the planes (column, row / 2, row % 2, plane),
//   so rows 2t and 2t+1 of lane t sit in two 512-byte slices and the 16-byte
//   reads of 8 lanes cover 128 contiguous bytes.  (A 16-byte wide box with
//   the 128-byte swizzle would put every row on its own 128-byte line, eight
//   times the space.)  A stage is copied to registers at its start and
//   immediately refilled.
// * Hacc uses an XOR layout of 8-byte units, conflict-free for the row pass
//   (each lane stores rows 2t, 2t+1 at one column pair) and for the column
//   pass (each lane reads columns 2t, 2t+1 of one row).
// * Every mbarrier wait is bounded (2 s); on expiry the warp records an
//   error word in the workspace, drains its outstanding copies and returns.
#include <type_traits>

#include "gspn_internal.h"
#include "gspn_lane.cuh"
#include "gspn_tma.cuh"
#include "gspn_tmem.cuh"

namespace gspn {

namespace {

using namespace lane;

// ---- kernel configuration ------------------------------------------------------------
constexpr int S = 64;          // H = W
constexpr int LPL = 32;        // lanes per line (2 positions per lane)
constexpr int NCW = 8;         // consumer warps per CTA (one plane each), one CTA per SM
constexpr int NST = 2;         // x/lambda ring stages per consumer warp
constexpr int NWS = 4;         // tap-weight stages, in shared memory (bulk copy) and in TMEM (64 columns)
constexpr int BOX = 1024;      // bytes per TMA box (one plane)
constexpr int SLICE = 512;     // the even or odd rows of a column chunk
constexpr int STAGE = 4 * BOX;
constexpr int HACC = S * S * 4;
constexpr int WCHUNK = 8 * S * 16;  // tap weights of 8 scan steps (8 table rows)
constexpr int WARP_BYTES = NST * STAGE + HACC;
constexpr int WRING = NCW * WARP_BYTES;              // offset of the weight ring
constexpr int BARS = WRING + NWS * WCHUNK;           // offset of the barriers
constexpr int NBAR = 2 * NCW * NST + 2 * NWS + 8 * NWS + 1;
constexpr int SMEM_BYTES = 1024 + BARS + 8 * NBAR + 16;  // + the TMEM address
constexpr int CHUNKS_PER_GROUP = 16;  // 8 column chunks + 8 row chunks
constexpr int NPW = NCW / 2;  // data producer warps, each feeding two consumer warps
constexpr int WW = NCW + NPW;  // the first of 4 tap-weight warps; warp WW + q writes lane quarter q
static_assert(WW % 4 == 0, "weight warp WW + q sits on lane quarter q");
constexpr int THREADS = (NCW + NPW + 4) * 32;
constexpr uint32_t TMEM_COLS = 512;  // first arrivals: 256 columns, then the tap-weight stages
constexpr uint32_t TW_COL = 256;     // first tap-weight column
static_assert(TW_COL + NWS * 64 <= TMEM_COLS, "tensor memory budget");
static_assert(SMEM_BYTES <= 232448, "shared memory budget");
static_assert(WARP_BYTES % 1024 == 0 && WCHUNK % 1024 == 0, "TMA destinations stay 1024-byte aligned");


// ---- weights pre-kernel ----------------------------------------------------------
// wtab[((b*2 + pass)*64 + s)*64 + p*32 + t] = (-w0_A, -w0_B, w2_A, w2_B) of line
// position j = 2t + p at scan step s, where pass 0 pairs A = left->right (line s
// = column s) with B = right->left (column 63-s), positions = rows; pass 1 pairs
// A = top->bottom (row s) with B = bottom->top (row 63-s), positions = columns.
template <typename T>
__device__ __forceinline__ void gate_pair(const T* lg, int pix, int j, float* w0, float* w2) {
    const float s0 = j > 0 ? sigmoidf(load_elt(lg, pix)) : 0.f;
    const float s1 = sigmoidf(load_elt(lg, S * S + pix));
    const float s2 = j < S - 1 ? sigmoidf(load_elt(lg, 2 * S * S + pix)) : 0.f;
    const float r = 1.f / (s0 + s1 + s2);
    *w0 = s0 * r;
    *w2 = s2 * r;
}

template <typename T>
__global__ void c64_weights_kernel(const T* __restrict__ logits, float4* __restrict__ wtab, int* err, int B) {
    const int idx = blockIdx.x * blockDim.x + threadIdx.x;
    if (idx == 0) *err = 0;
    if (idx >= B * 2 * S * S) return;
    const int j = idx & 63, s = (idx >> 6) & 63, pass = (idx >> 12) & 1, b = idx >> 13;
    const int slotA = pass ? 0 : 2, slotB = pass ? 1 : 3;
    const int pixA = pass ? s * S + j : j * S + s;
    const int pixB = pass ? (S - 1 - s) * S + j : j * S + (S - 1 - s);
    float w0a, w2a, w0b, w2b;
    gate_pair(logits + (size_t)(slotA * B + b) * 3 * S * S, pixA, j, &w0a, &w2a);
    gate_pair(logits + (size_t)(slotB * B + b) * 3 * S * S, pixB, j, &w0b, &w2b);
    const int t = j >> 1, p = j & 1;
    wtab[((size_t)(b * 2 + pass) * S + s) * S + p * LPL + t] = make_float4(-w0a, -w0b, w2a, w2b);
}

// One scan step for one lane: 2 positions, two directions packed in float2.
// base[p] = h[p] + lambda x (both directions), w[p] = (-w0_A, -w0_B, w2_A, w2_B).
__device__ __forceinline__ void scan_core(float2 (&h)[2], const float2 (&base)[2], const float4 (&w)[2]) {
    float2 hl, hr;
    hl.x = __shfl_up_sync(FULL, h[1].x, 1);
    hl.y = __shfl_up_sync(FULL, h[1].y, 1);
    hr.x = __shfl_down_sync(FULL, h[0].x, 1);
    hr.y = __shfl_down_sync(FULL, h[0].y, 1);
    const float2 D0 = sub2(h[0], hl), D1 = sub2(h[1], h[0]), D2 = sub2(hr, h[1]);
    const float2 v0 = __ffma2_rn(make_float2(w[0].z, w[0].w), D1, base[0]);
    const float2 v1 = __ffma2_rn(make_float2(w[1].z, w[1].w), D2, base[1]);
    h[0] = __ffma2_rn(make_float2(w[0].x, w[0].y), D0, v0);
    h[1] = __ffma2_rn(make_float2(w[1].x, w[1].y), D1, v1);
}

struct C64Args {
    const float4* wtab;
    __nv_bfloat16* out;
    int* err;
    int B, C, seg;
    int groups;  // B * C / 8 groups of 8 consecutive planes (one batch image each)
    uint64_t limit;  // bound of every wait on data, a stage or another warp (ns)
    int stall;       // test hook: consumer warp 0 of CTA 0 first waits on a barrier nothing completes
};

template <bool LOCAL>
__global__ void __launch_bounds__(THREADS, 1)
    c64_fwd_kernel(const __grid_constant__ CUtensorMap tm_xc, const __grid_constant__ CUtensorMap tm_lc,
                   const __grid_constant__ CUtensorMap tm_xr, const __grid_constant__ CUtensorMap tm_lr,
                   const C64Args a) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char* const smem = smem_raw + ((1024u - (tma::smem_u32(smem_raw) & 1023u)) & 1023u);
    const uint32_t sbase = tma::smem_u32(smem);
    const int warp = threadIdx.x >> 5, t = threadIdx.x & 31;
    const uint32_t xfull0 = sbase + BARS;                  // [warp][stage] "data landed"
    const uint32_t xempty0 = xfull0 + 8 * NCW * NST;       // [warp][stage] "data read"
    const uint32_t wfull0 = xempty0 + 8 * NCW * NST;       // [stage] weight chunk in shared memory
    const uint32_t wempty0 = wfull0 + 8 * NWS;             // [stage] the 4 weight warps have read it
    const uint32_t tfull0 = wempty0 + 8 * NWS;             // [stage][quarter] weight chunk in TMEM
    const uint32_t tempty0 = tfull0 + 8 * 4 * NWS;         // [stage][quarter] both consumers have loaded it
    const uint32_t done0 = tempty0 + 8 * 4 * NWS;          // every warp is done with the tensor memory
    uint32_t* const tslot = reinterpret_cast<uint32_t*>(smem + BARS + 8 * NBAR);
    if ((int)blockIdx.x >= a.groups) return;

    if (threadIdx.x == 0) {
        for (int s = 0; s < NCW * NST; ++s) {
            tma::mbar_init(xfull0 + 8 * s, 1);
            tma::mbar_init(xempty0 + 8 * s, 32);
        }
        for (int s = 0; s < NWS; ++s) {
            tma::mbar_init(wfull0 + 8 * s, 1);
            tma::mbar_init(wempty0 + 8 * s, 4);
        }
        for (int s = 0; s < 4 * NWS; ++s) {
            tma::mbar_init(tfull0 + 8 * s, 1);
            tma::mbar_init(tempty0 + 8 * s, 2);
        }
        tma::mbar_init(done0, NCW + 4);
        tma::fence_barrier_init();
    }
    if (warp == 0) {  // consumer warp 0 owns the CTA's 512 TMEM columns
        tmem::alloc(tma::smem_u32(tslot), TMEM_COLS);
        tmem::relinquish();
    }
    tmem::fence_before();
    __syncthreads();
    tmem::fence_after();
    const uint32_t taddr = *tslot;

    const int ngroups_here = (a.groups - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x;
    const int nchunks = ngroups_here * CHUNKS_PER_GROUP;

    const int BC = a.B * a.C;

    // ---------------- tap-weight warps ----------------
    // Lane 0 of weight warp 0 keeps NWS chunks of the tap-weight table in
    // flight into shared memory: chunk c (table rows 8*(c%16) .. +7 of the
    // group's image) into stage c % NWS, refilled with chunk c + NWS once all
    // four weight warps have read it.  Weight warp q writes chunk c into TMEM
    // stage c % NWS of lane quarter q once both consumers of the quarter have
    // loaded what it held: lane t takes the 16 bytes of positions p = 0, 1 of
    // each step e (table entry p*32 + t of row e) into columns 8e + 4p .. +3.
    if (warp >= WW) {
        const int qw = warp - WW;
        const uint32_t tq = taddr + ((uint32_t)(32 * qw) << 16) + TW_COL;
        auto fetch = [&](int c) {
            const int group = (int)blockIdx.x + (c / CHUNKS_PER_GROUP) * (int)gridDim.x;
            const int b = (8 * group) / a.C, ws = c % NWS;
            const float4* src = a.wtab + ((size_t)b * 2 * S + 8 * (c % CHUNKS_PER_GROUP)) * S;
            tma::mbar_expect_tx(wfull0 + 8 * ws, WCHUNK);
            tma::load_1d(sbase + WRING + ws * WCHUNK, src, WCHUNK, wfull0 + 8 * ws);
        };
        const bool feeder = qw == 0 && t == 0;
        int issued = 0;
        if (feeder)
            for (; issued < NWS && issued < nchunks; ++issued) fetch(issued);
        bool ok = true;
        for (int c = 0; c < nchunks; ++c) {
            const int ws = c % NWS;
            const uint32_t par = (uint32_t)(c / NWS) & 1u;
            const bool okw = tma::mbar_wait(wfull0 + 8 * ws, par, a.limit) &&
                             tma::mbar_wait(tempty0 + 8 * (ws * 4 + qw), par ^ 1u, a.limit);
            if (!__all_sync(FULL, okw)) {
                ok = false;
                break;
            }
            const unsigned char* src = smem + WRING + ws * WCHUNK + t * 16;
            tmem::fence_after();
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                uint32_t v[32];
#pragma unroll
                for (int e = 0; e < 4; ++e)
#pragma unroll
                    for (int p = 0; p < 2; ++p) {
                        const uint4 w = lds128(src + (4 * hh + e) * 1024 + p * 512);
                        v[e * 8 + p * 4 + 0] = w.x;
                        v[e * 8 + p * 4 + 1] = w.y;
                        v[e * 8 + p * 4 + 2] = w.z;
                        v[e * 8 + p * 4 + 3] = w.w;
                    }
                tmem::st_x32(tq + 64u * (uint32_t)ws + 32u * (uint32_t)hh, v);
            }
            // the shared stage is read: hand it back to the feeder
            tma::fence_proxy_async();
            __syncwarp();
            if (t == 0) tma::mbar_arrive(wempty0 + 8 * ws);
            tmem::wait_st();
            tmem::fence_before();
            __syncwarp();
            if (t == 0) tma::mbar_arrive(tfull0 + 8 * (ws * 4 + qw));
            if (feeder && issued < nchunks) {
                if (!tma::mbar_wait(wempty0 + 8 * ws, par, a.limit)) {
                    ok = false;
                } else {
                    fetch(issued++);
                }
            }
            if (!__all_sync(FULL, ok)) break;
        }
        // no bulk copy of the feeder is in flight when the CTA exits
        if (feeder)
            for (int c = 0; c < issued; ++c)
                if (c + NWS >= issued) tma::mbar_wait(wfull0 + 8 * (c % NWS), (c / NWS) & 1, 100000000ull);
        if (!ok && t == 0) atomicExch(a.err, 1);
        tmem::wait_st();
        tmem::fence_before();
        __syncwarp();
        if (t == 0) tma::mbar_arrive(done0);
        return;
    }

    // ---------------- data producer warps ----------------
    // Lane 0 of producer warp p streams the x / lambda chunks of consumer warps
    // 2p and 2p+1: chunk kk of warp w (plane 8*group + w of group blockIdx.x +
    // (kk/16)*gridDim.x; chunk kk%16: 0..7 column chunks, 8..15 row chunks;
    // lambda plane (slot, b, c) at slot*B*C + plane) goes to stage kk % NST of the
    // warp's ring once the warp has read what the stage held.
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
                const int local = kk % CHUNKS_PER_GROUP, st = kk % NST;
                for (int w = 2 * pw; w < 2 * pw + 2; ++w) {
                    if (!tma::mbar_wait(xempty0 + 8 * (w * NST + st), ((kk / NST) & 1) ^ 1, a.limit)) {
                        ok = false;
                        break;
                    }
                    const int plane = 8 * group + w;
                    const uint32_t dst = sbase + w * WARP_BYTES + st * STAGE, bar = xfull0 + 8 * (w * NST + st);
                    tma::mbar_expect_tx(bar, STAGE);
                    if (local < 8) {
                        const int q = local;
                        // x and lambda(left->right) at columns 8q.., x and lambda(right->left) at
                        // 8(7-q)..; all 64 rows through the (column, row/2, row%2) view, so row
                        // 2t+p lands in slice p at t*16
                        tma::load_4d(dst + 0 * BOX, &tm_xc, 8 * q, 0, 0, plane, bar);
                        tma::load_4d(dst + 1 * BOX, &tm_lc, 8 * q, 0, 0, 2 * BC + plane, bar);
                        tma::load_4d(dst + 2 * BOX, &tm_xc, 8 * (7 - q), 0, 0, plane, bar);
                        tma::load_4d(dst + 3 * BOX, &tm_lc, 8 * (7 - q), 0, 0, 3 * BC + plane, bar);
                    } else {
                        const int q = local - 8;
                        // x and lambda(top->bottom) at rows 8q.., x and lambda(bottom->top) at rows 56-8q..
                        tma::load_3d(dst + 0 * BOX, &tm_xr, 0, 8 * q, plane, bar);
                        tma::load_3d(dst + 1 * BOX, &tm_lr, 0, 8 * q, 0 * BC + plane, bar);
                        tma::load_3d(dst + 2 * BOX, &tm_xr, 0, 56 - 8 * q, plane, bar);
                        tma::load_3d(dst + 3 * BOX, &tm_lr, 0, 56 - 8 * q, 1 * BC + plane, bar);
                    }
                }
            }
            if (!ok) atomicExch(a.err, 1);
        }
        return;
    }

    // ---------------- consumer warps: one plane each ----------------
    unsigned char* const ringp = smem + warp * WARP_BYTES;
    unsigned char* const haccp = ringp + NST * STAGE;
    const uint32_t bar0 = xfull0 + 8 * NST * warp, ebar0 = xempty0 + 8 * NST * warp;
    const int segmask = a.seg - 1;  // seg divides 64, so it is a power of two

    int k = 0;            // next chunk to consume (same sequence for data and weights)
    int stage = 0;        // k % NST
    uint32_t phase = 0;   // bit s: parity of the next completion of data stage s
    auto fail = [&]() {
        if (t == 0) atomicExch(a.err, 1);
        tmem::wait_st();  // no TMEM access outlives the warp
        tmem::wait_ld_all();
        // drain every data copy that may still be in flight, with a short bound
        for (int kk = k; kk < k + NST && kk < nchunks; ++kk)
            tma::mbar_wait(bar0 + 8 * (kk % NST), (kk / NST) & 1, 100000000ull);
    };

    // Tap weights are read two steps at a time, one pair ahead: at the even
    // step e of chunk c a warp issues the TMEM load of steps e+2, e+3 (16
    // columns) and waits for it after step e+1's arithmetic.  At step 6 every
    // load of the chunk has completed, so the warp hands the stage back (one
    // arrival per warp) and loads steps 0, 1 of chunk c+1 once the quarter's
    // weight warp has written it.  Data stages are copied to registers whole at the
    // chunk's start.
    const uint32_t twq = taddr + ((uint32_t)(32 * (warp & 3)) << 16) + TW_COL;
    uint32_t wcur[16] = {}, wnxt[16];  // taps of steps (e, e+1) and of the next pair, 8 columns per step
    auto wissue = [&](int c, int e) -> bool {
        if ((e & 1) == 0) {
            if (e < 6) {
                tmem::ld_x16(twq + 64u * (uint32_t)(c % NWS) + 8u * (uint32_t)(e + 2), wnxt);
                return true;
            }
            tmem::fence_before();
            __syncwarp();
            if (t == 0) tma::mbar_arrive(tempty0 + 8 * ((c % NWS) * 4 + (warp & 3)));
            if (c + 1 < nchunks) {
                const bool okw =
                    tma::mbar_wait(tfull0 + 8 * (((c + 1) % NWS) * 4 + (warp & 3)), ((c + 1) / NWS) & 1, a.limit);
                if (!__all_sync(FULL, okw)) return false;
                tmem::fence_after();
                tmem::ld_x16(twq + 64u * (uint32_t)((c + 1) % NWS), wnxt);
            }
        }
        return true;
    };
    // the taps of step e as the (-w0_A, -w0_B, w2_A, w2_B) of positions 2t, 2t+1
    auto wget = [&](int e, float4 (&w)[2]) {
        const int o = (e & 1) * 8;
        w[0] = make_float4(__uint_as_float(wcur[o]), __uint_as_float(wcur[o + 1]), __uint_as_float(wcur[o + 2]),
                           __uint_as_float(wcur[o + 3]));
        w[1] = make_float4(__uint_as_float(wcur[o + 4]), __uint_as_float(wcur[o + 5]), __uint_as_float(wcur[o + 6]),
                           __uint_as_float(wcur[o + 7]));
    };
    // after the odd step: the next pair has arrived
    auto wturn = [&](int e) {
        if (e & 1) {
            tmem::wait_ld16(wnxt);
#pragma unroll
            for (int i = 0; i < 16; ++i) wcur[i] = wnxt[i];
        }
    };
    auto acquire = [&]() -> bool {
        const bool ok = tma::mbar_wait(bar0 + 8 * stage, (phase >> stage) & 1u, a.limit);
        return __all_sync(FULL, ok);
    };
    // the stage is in registers: hand it back to its producer
    auto release = [&]() {
        tma::fence_proxy_async();  // this lane's reads of the stage come before its refill
        tma::mbar_arrive(ebar0 + 8 * stage);
        phase ^= 1u << stage;
        ++k;
        stage = stage == NST - 1 ? 0 : stage + 1;
    };

    // Row pass: lane t owns rows 2t, 2t+1 (Hacc unit XOR key t & 15); row 2t + p
    // of a column chunk sits at p*512 + t*16.
    unsigned char* const hrow = haccp + 2 * t * 256;
    // First arrivals of a pass (its steps 0..31) wait in TMEM for the second:
    // lane t of lane quarter warp % 4, 128 columns from 128 * (warp / 4); a half
    // chunk (4 steps) is 16 columns [step][position][direction].
    const uint32_t tcol = taddr + ((uint32_t)(32 * (warp & 3)) << 16) + 128u * (uint32_t)(warp >> 2);
    const uint32_t tk8 = (uint32_t)(t & 15) << 3;
    const uint32_t t8 = (uint32_t)t << 3;
    float2 h[2];
    __nv_bfloat16* outp = nullptr;

    // Four column chunks of the row pass: left->right (x) and right->left (y).
    // SECOND: the chunks q = 4..7, where both directions are the second to reach
    // their columns and add to Hacc.
    auto row_half = [&](auto second) -> bool {
        constexpr bool SECOND = decltype(second)::value;
        for (int qq = 0; qq < 4; ++qq) {
            const int q = SECOND ? qq + 4 : qq;
            const int c = k;
            if (!acquire()) return false;
            const unsigned char* st = ringp + stage * STAGE + t * 16;
            uint4 XA[2], LA[2], XB[2], LB[2];
#pragma unroll
            for (int p = 0; p < 2; ++p) {
                XA[p] = lds128(st + 0 * BOX + p * SLICE);
                LA[p] = lds128(st + 1 * BOX + p * SLICE);
                XB[p] = lds128(st + 2 * BOX + p * SLICE);
                LB[p] = lds128(st + 3 * BOX + p * SLICE);
            }
            release();
            const uint32_t q8 = (uint32_t)(4 * q) << 3;
            float2 prev[2];
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                uint32_t tv[16];  // first arrivals of a half chunk: [step][position][direction]
                if (SECOND) {
                    // the first arrivals these steps meet were made at steps 63-s:
                    // half 1-hh of chunk 7-q
                    tmem::ld_x16(tcol + 32 * (7 - q) + 16 * (1 - hh), tv);
                    tmem::wait_ld16(tv);
                }
#pragma unroll
                for (int ee = 0; ee < 4; ++ee) {
                    const int e = 4 * hh + ee;
                    if (LOCAL && ((8 * q + e) & segmask) == 0) h[0] = h[1] = make_float2(0.f, 0.f);
                    // left->right reads column 8q+e = element e of the A chunk; right->left
                    // column 63-8q-e = element 7-e of the B chunk
                    float2 base[2];
#pragma unroll
                    for (int p = 0; p < 2; ++p) {
                        base[p].x = fma_bf(e & 1, word_of(LA[p], e >> 1), word_of(XA[p], e >> 1), h[p].x);
                        base[p].y = fma_bf((7 - e) & 1, word_of(LB[p], (7 - e) >> 1), word_of(XB[p], (7 - e) >> 1),
                                           h[p].y);
                    }
                    if (!wissue(c, e)) return false;
                    {
                        float4 wc[2];
                        wget(e, wc);
                        scan_core(h, base, wc);
                    }
                    wturn(e);
                    if constexpr (!SECOND) {
#pragma unroll
                        for (int p = 0; p < 2; ++p) {
                            tv[ee * 4 + p * 2] = __float_as_uint(h[p].x);
                            tv[ee * 4 + p * 2 + 1] = __float_as_uint(h[p].y);
                        }
                    } else {
                        // left->right at column s meets right->left's first arrival there
                        // (element 3-ee of the loaded half), right->left at column 63-s
                        // meets left->right's: the completed row sums
                        float2 sum[2];
#pragma unroll
                        for (int p = 0; p < 2; ++p)
                            sum[p] = __fadd2_rn(h[p], make_float2(__uint_as_float(tv[(3 - ee) * 4 + p * 2 + 1]),
                                                                  __uint_as_float(tv[(3 - ee) * 4 + p * 2])));
                        if (e & 1) {
                            // left->right covers columns s-1, s (unit s/2 = 4q + e/2), right->left
                            // columns 63-s, 64-s (unit 31 - (4q + e/2)); XOR with the row key
                            const uint32_t oA = (q8 + (uint32_t)((e >> 1) << 3)) ^ tk8;
                            const uint32_t oB = oA ^ (31u << 3);
#pragma unroll
                            for (int p = 0; p < 2; ++p) {
                                sts64f(hrow + p * 256 + oA, make_float2(prev[p].x, sum[p].x));
                                sts64f(hrow + p * 256 + oB, make_float2(sum[p].y, prev[p].y));
                            }
                        } else {
                            prev[0] = sum[0];
                            prev[1] = sum[1];
                        }
                    }
                }
                if (!SECOND) tmem::st_x16(tcol + 32 * q + 16 * hh, tv);
            }
        }
        return true;
    };

    // Four row chunks of the column pass: top->bottom (x) and bottom->top (y).
    // SECOND: the chunks q = 4..7, which complete their pixels and store them.
    auto col_half = [&](auto second) -> bool {
        constexpr bool SECOND = decltype(second)::value;
        for (int qq = 0; qq < 4; ++qq) {
            const int q = SECOND ? qq + 4 : qq;
            const int c = k;
            if (!acquire()) return false;
            const unsigned char* st = ringp + stage * STAGE + t * 4;
            uint32_t XA[8], LA[8], XB[8], LB[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                XA[e] = lds32(st + 0 * BOX + e * 128);
                LA[e] = lds32(st + 1 * BOX + e * 128);
                XB[e] = lds32(st + 2 * BOX + (7 - e) * 128);
                LB[e] = lds32(st + 3 * BOX + (7 - e) * 128);
            }
            release();
            // rows s = 8q + e (top->bottom) and 63 - s (bottom->top); the Hacc unit key
            // of row s is ((4q) & 15) + e/2, that of row 63 - s is 15 minus it
            unsigned char* const hA = haccp + 8 * q * 256;
            unsigned char* const hB = haccp + (S - 1 - 8 * q) * 256;
            const uint32_t k8 = (uint32_t)((4 * q) & 15) << 3;
            __nv_bfloat16* const oA_row = outp + (8 * q) * S;
            __nv_bfloat16* const oB_row = outp + (S - 1 - 8 * q) * S;
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                uint32_t tv[16];  // first arrivals of a half chunk: [step][top->bottom, bottom->top][position]
                if (SECOND) {
                    tmem::ld_x16(tcol + 32 * (7 - q) + 16 * (1 - hh), tv);
                    tmem::wait_ld16(tv);
                }
#pragma unroll
                for (int ee = 0; ee < 4; ++ee) {
                    const int e = 4 * hh + ee;
                    if (LOCAL && ((8 * q + e) & segmask) == 0) h[0] = h[1] = make_float2(0.f, 0.f);
                    float2 base[2];
                    base[0].x = fma_bf_lo(LA[e], XA[e], h[0].x);
                    base[1].x = fma_bf_hi(LA[e], XA[e], h[1].x);
                    base[0].y = fma_bf_lo(LB[e], XB[e], h[0].y);
                    base[1].y = fma_bf_hi(LB[e], XB[e], h[1].y);
                    if (!wissue(c, e)) return false;
                    {
                        float4 wc[2];
                        wget(e, wc);
                        scan_core(h, base, wc);
                    }
                    wturn(e);
                    if (!SECOND) {
                        // first arrival of this pass: the row sum of the pixel plus this
                        // direction's value, parked in TMEM
                        const uint32_t oA = (k8 + (uint32_t)((e >> 1) << 3)) ^ t8;
                        const uint32_t oB = oA ^ (15u << 3);
                        const float2 vA = __fadd2_rn(lds64f(hA + e * 256 + oA), make_float2(h[0].x, h[1].x));
                        const float2 vB = __fadd2_rn(lds64f(hB - e * 256 + oB), make_float2(h[0].y, h[1].y));
                        tv[ee * 4 + 0] = __float_as_uint(vA.x);
                        tv[ee * 4 + 1] = __float_as_uint(vA.y);
                        tv[ee * 4 + 2] = __float_as_uint(vB.x);
                        tv[ee * 4 + 3] = __float_as_uint(vB.y);
                    } else {
                        // second arrival: top->bottom at row s meets bottom->top's first
                        // arrival there (element 3-ee of the loaded half), and vice versa
                        const int f = (3 - ee) * 4;
                        const float2 vA = __fadd2_rn(make_float2(__uint_as_float(tv[f + 2]), __uint_as_float(tv[f + 3])),
                                                     make_float2(h[0].x, h[1].x));
                        const float2 vB = __fadd2_rn(make_float2(__uint_as_float(tv[f]), __uint_as_float(tv[f + 1])),
                                                     make_float2(h[0].y, h[1].y));
                        stg_cs32(oA_row + e * S, pack_bf2(vA.x, vA.y));
                        stg_cs32(oB_row - e * S, pack_bf2(vB.x, vB.y));
                    }
                }
                if (!SECOND) tmem::st_x16(tcol + 32 * q + 16 * hh, tv);
            }
        }
        return true;
    };

    bool ok = true;
    if (a.stall && blockIdx.x == 0 && warp == 0) {
        // test hook: phase 0 of done0 needs this warp's own final arrival, so
        // this wait can only run out; the kernel then takes its error path
        ok = __all_sync(FULL, tma::mbar_wait(done0, 0, a.limit));
    }
    if (ok && nchunks > 0) {
        const bool okw = tma::mbar_wait(tfull0 + 8 * (warp & 3), 0, a.limit);
        ok = __all_sync(FULL, okw);
        if (ok) {
            tmem::fence_after();
            tmem::ld_x16(twq, wcur);
            tmem::wait_ld16(wcur);
        }
    }
    for (int group = blockIdx.x; ok && group < a.groups; group += gridDim.x) {
        outp = a.out + (size_t)(8 * group + warp) * S * S + 2 * t;
        h[0] = h[1] = make_float2(0.f, 0.f);
        ok = row_half(std::false_type{});
        tmem::wait_st();  // the second half reads what the first half parked
        ok = ok && row_half(std::true_type{});
        __syncwarp();
        h[0] = h[1] = make_float2(0.f, 0.f);
        ok = ok && col_half(std::false_type{});
        tmem::wait_st();
        ok = ok && col_half(std::true_type{});
        __syncwarp();
    }
    if (!ok) fail();
    // this warp no longer touches the tensor memory; warp 0 frees it after all
    // consumers and the weight warps
    tmem::wait_st();
    tmem::wait_ld_all();
    tmem::fence_before();
    __syncwarp();
    if (t == 0) tma::mbar_arrive(done0);
    if (warp == 0) {
        if (!tma::mbar_wait(done0, 0, 10 * tma::kTimeoutNs) && t == 0) atomicExch(a.err, 1);
        __syncwarp();
        tmem::fence_after();
        tmem::dealloc(taddr, TMEM_COLS);
    }
}

// ---- host side ----------------------------------------------------------------------
// 3-D view (column, row, plane) of a stack of 64x64 bf16 planes; one plane per
// box of box_c columns x box_r rows (every row_step-th row).
bool make_map(CUtensorMap* m, const void* base, uint64_t planes, uint32_t box_c, uint32_t box_r, uint32_t row_step,
              CUtensorMapL2promotion promo) {
    EncodeTiledFn fn = encode_tiled();
    if (!fn) return false;
    const cuuint64_t dims[3] = {S, S, planes};
    const cuuint64_t strides[2] = {S * 2, S * S * 2};
    const cuuint32_t box[3] = {box_c, box_r, 1};
    const cuuint32_t es[3] = {1, row_step, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, promo,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Row-pass view of the same planes: (column, row / 2, row % 2, plane); one box =
// 8 columns of all 64 rows, laid out [row % 2][row / 2][8 columns], so the
// 16-byte reads of a warp (lane t: rows 2t, 2t+1) are conflict-free.
bool make_map_cols(CUtensorMap* m, const void* base, uint64_t planes) {
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

template <bool LOCAL>
gspn_status launch_c64(const DeviceInfo& dev, const CUtensorMap& xc, const CUtensorMap& lc, const CUtensorMap& xr,
                       const CUtensorMap& lr, const C64Args& a, cudaStream_t s) {
    const void* fn = (const void*)c64_fwd_kernel<LOCAL>;
    cudaError_t e = ensure_smem_attr(fn, SMEM_BYTES, LOCAL ? 9 : 8);
    if (e != cudaSuccess) return GSPN_ERR_CUDA;
    const int grid = a.groups < dev.sm_count ? a.groups : dev.sm_count;
    c64_fwd_kernel<LOCAL><<<grid, THREADS, SMEM_BYTES, s>>>(xc, lc, xr, lr, a);
    return cudaGetLastError() == cudaSuccess ? GSPN_OK : GSPN_ERR_CUDA;
}

}  // namespace

bool c64_eligible(const Problem& p) {
    return p.d.dtype == GSPN_BF16 && p.g.shared && p.d.dir_mask == 15u && p.g.H == S && p.g.W == S &&
           p.g.C % 8 == 0 && p.planes <= 0x7fffffff / 4 && encode_tiled() != nullptr;
}

size_t c64_fwd_workspace(const Problem& p) {
    return kWsAlign + align_up((size_t)p.g.B * 2 * S * S * sizeof(float4), kWsAlign);
}

gspn_status c64_fwd(const Problem& p, const DeviceInfo& dev, const void* x, const void* logits, const void* lam,
                    void* out, void* ws, cudaStream_t s) {
    CUtensorMap xc, lc, xr, lr;
    const uint64_t BC = (uint64_t)p.planes;
    // column chunks: 8 columns x every other row (32 rows); row chunks: 64 columns x 8 rows
    if (!make_map_cols(&xc, x, BC) || !make_map_cols(&lc, lam, 4 * BC) ||
        !make_map(&xr, x, BC, 64, 8, 1, CU_TENSOR_MAP_L2_PROMOTION_L2_128B) ||
        !make_map(&lr, lam, 4 * BC, 64, 8, 1, CU_TENSOR_MAP_L2_PROMOTION_L2_128B))
        return GSPN_ERR_UNSUPPORTED;
    char* w = static_cast<char*>(ws);
    C64Args a;
    a.err = reinterpret_cast<int*>(w);
    a.wtab = reinterpret_cast<const float4*>(w + kWsAlign);
    a.out = static_cast<__nv_bfloat16*>(out);
    a.B = p.g.B;
    a.C = p.g.C;
    a.seg = S / p.g.groups;
    a.groups = (int)(p.planes / 8);
    const WaitCfg wc = wait_cfg();
    a.limit = wc.limit_ns;
    a.stall = wc.stall;
    const int nw = p.g.B * 2 * S * S;
    c64_weights_kernel<__nv_bfloat16><<<(nw + 255) / 256, 256, 0, s>>>(
        static_cast<const __nv_bfloat16*>(logits), const_cast<float4*>(a.wtab), a.err, p.g.B);
    if (cudaGetLastError() != cudaSuccess) return GSPN_ERR_CUDA;
    return p.g.groups > 1 ? launch_c64<true>(dev, xc, lc, xr, lr, a, s) : launch_c64<false>(dev, xc, lc, xr, lr, a, s);
}

// ---- allocation-free entry (gspn_fwd_noalloc) ------------------------------------
// Fixed scratch of the forward for callers that cannot allocate device memory:
// the error word and the tap-weight table of up to kNoAllocMaxBatch batch
// images (4 MiB + 256 bytes).  Every GPU that loads the library holds it until
// the process exits; all calls share it (the weights pre-kernel rewrites both
// the error word and every table row a call reads).
namespace {
constexpr int kNoAllocMaxBatch = 32;
constexpr size_t kNoAllocBytes = kWsAlign + (size_t)kNoAllocMaxBatch * 2 * S * S * sizeof(float4);
__device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocBytes];

// Device address of the array in the current context.  In host code the
// array's name is only a host-side stand-in.  The address is looked up on
// every call (a host-side table lookup once the module is loaded), so a
// context that was torn down and recreated -- cudaDeviceReset, or a primary
// context released and retained again -- never sees a stale address.  With
// lazy module loading the first call on a device also loads the module, which
// places the array: make that first call before any stream capture begins.
void* noalloc_scratch() {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess) return nullptr;
    return ptr;
}
}  // namespace

gspn_status c64_fwd_noalloc(const Problem& p, const DeviceInfo& dev, const void* x, const void* logits,
                            const void* lam, void* out, cudaStream_t s) {
    if (!c64_eligible(p)) return GSPN_ERR_UNSUPPORTED;
    if (p.g.B > kNoAllocMaxBatch || c64_fwd_workspace(p) > kNoAllocBytes) return GSPN_ERR_SCRATCH_LIMIT;
    void* ptr = noalloc_scratch();
    if (!ptr) return GSPN_ERR_CUDA;
    return c64_fwd(p, dev, x, logits, lam, out, ptr, s);
}

gspn_status c64_noalloc_status(cudaStream_t s) {
    void* ptr = noalloc_scratch();
    if (!ptr) return GSPN_ERR_CUDA;
    int v = 0;
    if (cudaMemcpyAsync(&v, ptr, sizeof(v), cudaMemcpyDeviceToHost, s) != cudaSuccess) return GSPN_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return GSPN_ERR_CUDA;
    return v ? GSPN_ERR_TIMEOUT : GSPN_OK;
}

}  // namespace gspn
