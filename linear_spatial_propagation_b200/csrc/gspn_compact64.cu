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
//   direction) -- w1 = 1 - w0 - w2 -- laid out in scan order, so that each
//   scan step reads one contiguous 512-byte row per warp; the main kernel
//   reads them through L1 (prefetched 8 steps ahead) for every channel.
// * One warp scans KC (2 when C is even, else 1) planes of one batch image:
//   32 lanes per 64-wide line, 2 positions per lane, the KC channels in the
//   same lane so that each step's tap weights are loaded once for all of
//   them; 8 / KC warps per SM.  The two directions of a pair (left->right with
//   right->left, top->bottom with bottom->top) advance together: lane values
//   are float2 (one direction per half) and the update is the packed fp32x2
//   FMA of sm_100; lambda*x is one mixed-precision FMA with bf16 inputs.
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
// * All x / lambda traffic is streamed by TMA into a per-warp ring of 4 KB
//   stages (8 scan steps each): column chunks (8 columns x 64 rows) for the
//   row pass and row chunks (64 columns x 8 rows) for the column pass.  A
//   column chunk is fetched as two boxes of every other row (row element
//   stride 2), so rows 2t and 2t+1 of lane t sit in two 512-byte slices and
//   the 16-byte reads of 8 lanes cover 128 contiguous bytes.  (A 16-byte wide
//   box with the 128-byte swizzle would put every row on its own 128-byte
//   line, eight times the space.)  A stage is copied to registers at its
//   start and immediately refilled, so NST stages per warp stay in flight.
// * Hacc uses an XOR layout of 8-byte units, conflict-free for the row pass
//   (each lane stores rows 2t, 2t+1 at one column pair) and for the column
//   pass (each lane reads columns 2t, 2t+1 of one row).
// * Every mbarrier wait is bounded (2 s); on expiry the warp records an
//   error word in the workspace, drains its outstanding copies and returns.
#include <type_traits>

#include "gspn_internal.h"
#include "gspn_tma.cuh"

namespace gspn {

namespace {

constexpr int S = 64;         // H = W
constexpr int LPL = 32;       // lanes per line (2 positions per lane)
constexpr int NST = 3;        // ring stages per warp
constexpr int SLICE = 512;    // bytes of one plane in one element-stride-2 column box
constexpr int HACC = S * S * 4;
constexpr int CHUNKS_PER_UNIT = 16;  // 8 column chunks + 8 row chunks
constexpr int SMEM_OPTIN = 232448;

// KC channels per lane (the tap weights of a step are loaded once for all of
// them); 8 / KC warps per CTA, one CTA per SM.
template <int KC>
struct Cfg {
    static constexpr int NWARP = 8 / KC;
    static constexpr int BOX = KC * 1024;           // bytes per tensor per stage (KC planes)
    static constexpr int STAGE = 4 * BOX;
    static constexpr int WARP_BYTES = NST * STAGE + KC * HACC;
    static constexpr int BAR_BYTES = 8 * NST;
    static constexpr int SMEM_BYTES = 1024 + NWARP * WARP_BYTES + NWARP * BAR_BYTES;
    static_assert(SMEM_BYTES <= SMEM_OPTIN, "shared memory budget");
    static_assert(WARP_BYTES % 1024 == 0, "per-warp regions keep TMA destinations 1024-byte aligned");
};

constexpr unsigned FULL = 0xffffffffu;

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

// ---- helpers ----------------------------------------------------------------------
// Shared memory is addressed through ordinary pointers into the dynamic
// shared array, so the compiler folds constant offsets into the accesses; the
// TMA-written data is read only after the mbarrier wait (an asm with a memory
// clobber), which orders these loads behind it.
__device__ __forceinline__ uint4 lds128(const unsigned char* p) { return *reinterpret_cast<const uint4*>(p); }
__device__ __forceinline__ uint32_t lds32(const unsigned char* p) { return *reinterpret_cast<const uint32_t*>(p); }
__device__ __forceinline__ float2 lds64f(const unsigned char* p) { return *reinterpret_cast<const float2*>(p); }
__device__ __forceinline__ void sts64f(unsigned char* p, float2 v) { *reinterpret_cast<float2*>(p) = v; }
__device__ __forceinline__ void stg_cs32(__nv_bfloat16* p, uint32_t v) {
    __stcs(reinterpret_cast<unsigned int*>(p), v);
}
__device__ __forceinline__ uint32_t pack_bf2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}
__device__ __forceinline__ uint32_t word_of(const uint4& v, int i) {
    return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w;
}

// a - b, exactly rounded (sm_100 has packed add and fma but no packed subtract)
__device__ __forceinline__ float2 sub2(float2 a, float2 b) { return __ffma2_rn(b, make_float2(-1.f, -1.f), a); }

// c + a*b with a, b the low / high bf16 halves of two 32-bit words: the bf16
// operands feed the fp32 FMA directly (mixed-precision fma of sm_100), exact
// products and one rounding, like the fp32 FMA of the widened values.
__device__ __forceinline__ float fma_bf_lo(uint32_t a, uint32_t b, float c) {
    float d;
    asm("{\n\t.reg .b16 a0, a1, b0, b1;\n\tmov.b32 {a0, a1}, %1;\n\tmov.b32 {b0, b1}, %2;\n\t"
        "fma.rn.f32.bf16 %0, a0, b0, %3;\n\t}"
        : "=f"(d) : "r"(a), "r"(b), "f"(c));
    return d;
}
__device__ __forceinline__ float fma_bf_hi(uint32_t a, uint32_t b, float c) {
    float d;
    asm("{\n\t.reg .b16 a0, a1, b0, b1;\n\tmov.b32 {a0, a1}, %1;\n\tmov.b32 {b0, b1}, %2;\n\t"
        "fma.rn.f32.bf16 %0, a1, b1, %3;\n\t}"
        : "=f"(d) : "r"(a), "r"(b), "f"(c));
    return d;
}
// `half` is a compile-time constant at every (unrolled) call site
__device__ __forceinline__ float fma_bf(int half, uint32_t a, uint32_t b, float c) {
    return half ? fma_bf_hi(a, b, c) : fma_bf_lo(a, b, c);
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

// Hacc byte offset of the 8-byte unit u (columns 2u, 2u+1) of row r.
__device__ __forceinline__ uint32_t hacc_off(int r, int u) {
    return (uint32_t)(r * 256 + ((u ^ ((r >> 1) & 15)) << 3));
}

struct C64Args {
    const float4* wtab;
    __nv_bfloat16* out;
    int* err;
    int B, C, seg;
    int units;  // B * C / KC units of KC consecutive planes
};

template <int KC, bool LOCAL>
__global__ void __launch_bounds__(Cfg<KC>::NWARP * 32, 1)
    c64_fwd_kernel(const __grid_constant__ CUtensorMap tm_xc, const __grid_constant__ CUtensorMap tm_lc,
                   const __grid_constant__ CUtensorMap tm_xr, const __grid_constant__ CUtensorMap tm_lr,
                   const C64Args a) {
    using K = Cfg<KC>;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char* const smem = smem_raw + ((1024u - (tma::smem_u32(smem_raw) & 1023u)) & 1023u);
    const uint32_t sbase = tma::smem_u32(smem);
    const int warp = threadIdx.x >> 5, t = threadIdx.x & 31;
    const uint32_t ring = sbase + warp * K::WARP_BYTES;        // shared-window address (TMA)
    unsigned char* const ringp = smem + warp * K::WARP_BYTES;  // same bytes, for loads
    unsigned char* const haccp = ringp + NST * K::STAGE;       // KC planes of fp32
    const uint32_t bar0 = sbase + K::NWARP * K::WARP_BYTES + warp * K::BAR_BYTES;
    const int wid = blockIdx.x * K::NWARP + warp;
    const int wstride = gridDim.x * K::NWARP;
    const int segmask = a.seg - 1;  // seg divides 64, so it is a power of two
    const int BC = a.B * a.C;
    if (wid >= a.units) return;

    if (t == 0) {
        for (int s = 0; s < NST; ++s) tma::mbar_init(bar0 + 8 * s, 1);
        tma::fence_barrier_init();
        tma::prefetch_map(&tm_xc);
        tma::prefetch_map(&tm_lc);
        tma::prefetch_map(&tm_xr);
        tma::prefetch_map(&tm_lr);
    }
    __syncwarp();

    // Issue chunk kk of this warp's sequence (lane 0 only): unit wid + (kk/16)*wstride
    // (planes KC*unit ..), chunk kk%16 of it (0..7: column chunks, 8..15: row
    // chunks).  lambda plane (slot, b, c) is slot*B*C + plane.
    auto issue = [&](int kk) {
        const int unit = wid + (kk / CHUNKS_PER_UNIT) * wstride;
        if (unit >= a.units) return;
        const int plane = KC * unit;
        const int local = kk % CHUNKS_PER_UNIT, st = kk % NST;
        const uint32_t dst = ring + st * K::STAGE, bar = bar0 + 8 * st;
        tma::mbar_expect_tx(bar, K::STAGE);
        if (local < 8) {
            const int q = local;
            // x and lambda(left->right) at columns 8q.., x and lambda(right->left) at
            // 8(7-q)..; rows r_lo, r_lo + 2, ... of the KC planes go to slice r_lo
            for (int r = 0; r < 2; ++r) {
                const uint32_t o = r * KC * SLICE;
                tma::load_3d(dst + 0 * K::BOX + o, &tm_xc, 8 * q, r, plane, bar);
                tma::load_3d(dst + 1 * K::BOX + o, &tm_lc, 8 * q, r, 2 * BC + plane, bar);
                tma::load_3d(dst + 2 * K::BOX + o, &tm_xc, 8 * (7 - q), r, plane, bar);
                tma::load_3d(dst + 3 * K::BOX + o, &tm_lc, 8 * (7 - q), r, 3 * BC + plane, bar);
            }
        } else {
            const int q = local - 8;
            // x and lambda(top->bottom) at rows 8q.., x and lambda(bottom->top) at rows 56-8q..
            tma::load_3d(dst + 0 * K::BOX, &tm_xr, 0, 8 * q, plane, bar);
            tma::load_3d(dst + 1 * K::BOX, &tm_lr, 0, 8 * q, 0 * BC + plane, bar);
            tma::load_3d(dst + 2 * K::BOX, &tm_xr, 0, 56 - 8 * q, plane, bar);
            tma::load_3d(dst + 3 * K::BOX, &tm_lr, 0, 56 - 8 * q, 1 * BC + plane, bar);
        }
    };

    if (t == 0)
        for (int kk = 0; kk < NST; ++kk) issue(kk);

    int k = 0;            // next chunk to consume
    int stage = 0;        // k % NST
    uint32_t phase = 0;   // bit s: parity of the next completion of stage s
    auto fail = [&]() {
        if (t == 0) atomicExch(a.err, 1);
        // drain every copy that may still be in flight, with a short bound
        for (int kk = k; kk < k + NST; ++kk) {
            const int unit = wid + (kk / CHUNKS_PER_UNIT) * wstride;
            if (unit < a.units) tma::mbar_wait(bar0 + 8 * (kk % NST), (kk / NST) & 1, 100000000ull);
        }
    };
    // wait for chunk k; false (for every lane) if any lane's wait timed out
    auto acquire = [&]() -> bool {
        const bool ok = tma::mbar_wait(bar0 + 8 * stage, (phase >> stage) & 1u);
        return __all_sync(FULL, ok);
    };
    // all lanes done reading the stage of chunk k: refill it with chunk k + NST
    auto release = [&]() {
        tma::fence_proxy_async();
        __syncwarp();
        if (t == 0) issue(k + NST);
        phase ^= 1u << stage;
        ++k;
        stage = stage == NST - 1 ? 0 : stage + 1;
    };

    // Tap weights: a unit's 128 scan steps (64 row-pass, then 64 column-pass)
    // are table rows b*128 + l.  wr[e] holds the taps of the step l with
    // l % 8 == e; right after step l uses them it is refilled with step l + 8,
    // which continues into the next unit of this warp.
    float4 wr[8][2];
    auto wbase = [&](int unit) -> const float4* {
        return a.wtab + (size_t)((KC * unit) / a.C) * 2 * S * S + t;
    };
    const float4* wu = wbase(wid);
    const float4* wn = wid + wstride < a.units ? wbase(wid + wstride) : wu;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        wr[e][0] = __ldg(wu + e * S);
        wr[e][1] = __ldg(wu + e * S + LPL);
    }
    // first table row of the refills issued by the chunk starting at unit step l0
    auto wnext = [&](int l0) -> const float4* { return l0 + 8 < 2 * S ? wu + (l0 + 8) * S : wn; };

    // Row pass: lane t owns rows 2t, 2t+1 of each of its KC planes (Hacc unit
    // XOR key t & 15); row 2t + p of plane c of a column chunk sits at
    // p*KC*512 + c*512 + t*16.
    unsigned char* const hrow = haccp + 2 * t * 256;
    const uint32_t tk8 = (uint32_t)(t & 15) << 3;
    const uint32_t t8 = (uint32_t)t << 3;
    float2 h[KC][2];
    __nv_bfloat16* outp = nullptr;

    // Four column chunks of the row pass: left->right (x) and right->left (y).
    // SECOND: the chunks q = 4..7, where both directions are the second to reach
    // their columns and add to Hacc.
    auto row_half = [&](auto second) -> bool {
        constexpr bool SECOND = decltype(second)::value;
        for (int qq = 0; qq < 4; ++qq) {
            const int q = SECOND ? qq + 4 : qq;
            if (!acquire()) return false;
            const unsigned char* st = ringp + stage * K::STAGE + t * 16;
            uint4 XA[KC][2], LA[KC][2], XB[KC][2], LB[KC][2];
#pragma unroll
            for (int c = 0; c < KC; ++c)
#pragma unroll
                for (int p = 0; p < 2; ++p) {
                    const int o = p * KC * SLICE + c * SLICE;
                    XA[c][p] = lds128(st + 0 * K::BOX + o);
                    LA[c][p] = lds128(st + 1 * K::BOX + o);
                    XB[c][p] = lds128(st + 2 * K::BOX + o);
                    LB[c][p] = lds128(st + 3 * K::BOX + o);
                }
            release();
            const float4* wp = wnext(8 * q);
            const uint32_t q8 = (uint32_t)(4 * q) << 3;
            float2 prev[KC][2];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                if (LOCAL && ((8 * q + e) & segmask) == 0) {
#pragma unroll
                    for (int c = 0; c < KC; ++c) h[c][0] = h[c][1] = make_float2(0.f, 0.f);
                }
                // left->right reads column 8q+e = element e of the A chunk; right->left
                // column 63-8q-e = element 7-e of the B chunk
#pragma unroll
                for (int c = 0; c < KC; ++c) {
                    float2 base[2];
#pragma unroll
                    for (int p = 0; p < 2; ++p) {
                        base[p].x = fma_bf(e & 1, word_of(LA[c][p], e >> 1), word_of(XA[c][p], e >> 1), h[c][p].x);
                        base[p].y = fma_bf((7 - e) & 1, word_of(LB[c][p], (7 - e) >> 1),
                                           word_of(XB[c][p], (7 - e) >> 1), h[c][p].y);
                    }
                    scan_core(h[c], base, wr[e]);
                }
                wr[e][0] = __ldg(wp + e * S);
                wr[e][1] = __ldg(wp + e * S + LPL);
                if (e & 1) {
                    // left->right covers columns s-1, s (unit s/2 = 4q + e/2), right->left
                    // columns 63-s, 64-s (unit 31 - (4q + e/2)); XOR with the row key
                    const uint32_t oA = (q8 + (uint32_t)((e >> 1) << 3)) ^ tk8;
                    const uint32_t oB = oA ^ (31u << 3);
#pragma unroll
                    for (int c = 0; c < KC; ++c)
#pragma unroll
                        for (int p = 0; p < 2; ++p) {
                            unsigned char* adA = hrow + c * HACC + p * 256 + oA;
                            unsigned char* adB = hrow + c * HACC + p * 256 + oB;
                            float2 vA = make_float2(prev[c][p].x, h[c][p].x);
                            float2 vB = make_float2(h[c][p].y, prev[c][p].y);
                            if (SECOND) {
                                vA = __fadd2_rn(vA, lds64f(adA));
                                vB = __fadd2_rn(vB, lds64f(adB));
                            }
                            sts64f(adA, vA);
                            sts64f(adB, vB);
                        }
                } else {
#pragma unroll
                    for (int c = 0; c < KC; ++c) {
                        prev[c][0] = h[c][0];
                        prev[c][1] = h[c][1];
                    }
                }
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
            if (!acquire()) return false;
            const unsigned char* st = ringp + stage * K::STAGE + t * 4;
            uint32_t XA[KC][8], LA[KC][8], XB[KC][8], LB[KC][8];
#pragma unroll
            for (int c = 0; c < KC; ++c)
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    XA[c][e] = lds32(st + 0 * K::BOX + c * 1024 + e * 128);
                    LA[c][e] = lds32(st + 1 * K::BOX + c * 1024 + e * 128);
                    XB[c][e] = lds32(st + 2 * K::BOX + c * 1024 + (7 - e) * 128);
                    LB[c][e] = lds32(st + 3 * K::BOX + c * 1024 + (7 - e) * 128);
                }
            release();
            const float4* wp = wnext(S + 8 * q);
            // rows s = 8q + e (top->bottom) and 63 - s (bottom->top); the Hacc unit key
            // of row s is ((4q) & 15) + e/2, that of row 63 - s is 15 minus it
            unsigned char* const hA = haccp + 8 * q * 256;
            unsigned char* const hB = haccp + (S - 1 - 8 * q) * 256;
            const uint32_t k8 = (uint32_t)((4 * q) & 15) << 3;
            __nv_bfloat16* const oA_row = outp + (8 * q) * S;
            __nv_bfloat16* const oB_row = outp + (S - 1 - 8 * q) * S;
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                if (LOCAL && ((8 * q + e) & segmask) == 0) {
#pragma unroll
                    for (int c = 0; c < KC; ++c) h[c][0] = h[c][1] = make_float2(0.f, 0.f);
                }
#pragma unroll
                for (int c = 0; c < KC; ++c) {
                    float2 base[2];
                    base[0].x = fma_bf_lo(LA[c][e], XA[c][e], h[c][0].x);
                    base[1].x = fma_bf_hi(LA[c][e], XA[c][e], h[c][1].x);
                    base[0].y = fma_bf_lo(LB[c][e], XB[c][e], h[c][0].y);
                    base[1].y = fma_bf_hi(LB[c][e], XB[c][e], h[c][1].y);
                    scan_core(h[c], base, wr[e]);
                }
                wr[e][0] = __ldg(wp + e * S);
                wr[e][1] = __ldg(wp + e * S + LPL);
                const uint32_t oA = (k8 + (uint32_t)((e >> 1) << 3)) ^ t8;
                const uint32_t oB = oA ^ (15u << 3);
#pragma unroll
                for (int c = 0; c < KC; ++c) {
                    unsigned char* adA = hA + c * HACC + e * 256 + oA;
                    unsigned char* adB = hB + c * HACC - e * 256 + oB;
                    const float2 vA = __fadd2_rn(lds64f(adA), make_float2(h[c][0].x, h[c][1].x));
                    const float2 vB = __fadd2_rn(lds64f(adB), make_float2(h[c][0].y, h[c][1].y));
                    if (!SECOND) {  // first arrival of this pass: keep the partial sum
                        sts64f(adA, vA);
                        sts64f(adB, vB);
                    } else {        // second arrival: the pixel is complete
                        stg_cs32(oA_row + c * S * S + e * S, pack_bf2(vA.x, vA.y));
                        stg_cs32(oB_row + c * S * S - e * S, pack_bf2(vB.x, vB.y));
                    }
                }
            }
        }
        return true;
    };

    for (int unit = wid; unit < a.units; unit += wstride) {
        outp = a.out + (size_t)(KC * unit) * S * S + 2 * t;
#pragma unroll
        for (int c = 0; c < KC; ++c) h[c][0] = h[c][1] = make_float2(0.f, 0.f);
        if (!row_half(std::false_type{}) || !row_half(std::true_type{})) { fail(); return; }
        __syncwarp();
#pragma unroll
        for (int c = 0; c < KC; ++c) h[c][0] = h[c][1] = make_float2(0.f, 0.f);
        if (!col_half(std::false_type{}) || !col_half(std::true_type{})) { fail(); return; }
        __syncwarp();
        wu = wn;
        wn = unit + 2 * wstride < a.units ? wbase(unit + 2 * wstride) : wu;
    }
}

// ---- host side ----------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static bool tried = false;
    if (!tried) {
        tried = true;
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

// 3-D view (column, row, plane) of a stack of 64x64 bf16 planes; boxes of
// box_c columns x box_r rows (every row_step-th row) x box_p planes.
bool make_map(CUtensorMap* m, const void* base, uint64_t planes, uint32_t box_c, uint32_t box_r, uint32_t row_step,
              uint32_t box_p, CUtensorMapL2promotion promo) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[3] = {S, S, planes};
    const cuuint64_t strides[2] = {S * 2, S * S * 2};
    const cuuint32_t box[3] = {box_c, box_r, box_p};
    const cuuint32_t es[3] = {1, row_step, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, promo,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int KC, bool LOCAL>
gspn_status launch_c64(const DeviceInfo& dev, const CUtensorMap& xc, const CUtensorMap& lc, const CUtensorMap& xr,
                       const CUtensorMap& lr, const C64Args& a, cudaStream_t s) {
    using K = Cfg<KC>;
    const void* fn = (const void*)c64_fwd_kernel<KC, LOCAL>;
    cudaError_t e = ensure_smem_attr(fn, K::SMEM_BYTES, 8 + 2 * (KC - 1) + (LOCAL ? 1 : 0));
    if (e != cudaSuccess) return GSPN_ERR_CUDA;
    int grid = dev.sm_count;
    const int need = (a.units + K::NWARP - 1) / K::NWARP;
    if (need < grid) grid = need;
    c64_fwd_kernel<KC, LOCAL><<<grid, K::NWARP * 32, K::SMEM_BYTES, s>>>(xc, lc, xr, lr, a);
    return cudaGetLastError() == cudaSuccess ? GSPN_OK : GSPN_ERR_CUDA;
}

}  // namespace

bool c64_eligible(const Problem& p) {
    return p.d.dtype == GSPN_BF16 && p.g.shared && p.d.dir_mask == 15u && p.g.H == S && p.g.W == S &&
           p.planes <= 0x7fffffff / 4 && encode_fn() != nullptr;
}

size_t c64_fwd_workspace(const Problem& p) {
    return kWsAlign + align_up((size_t)p.g.B * 2 * S * S * sizeof(float4), kWsAlign);
}

gspn_status c64_fwd(const Problem& p, const DeviceInfo& dev, const void* x, const void* logits, const void* lam,
                    void* out, void* ws, cudaStream_t s) {
    // two channels per lane when C is even (the pair shares one batch image)
    const int kc = (p.g.C % 2 == 0) ? 2 : 1;
    CUtensorMap xc, lc, xr, lr;
    const uint64_t BC = (uint64_t)p.planes;
    // column chunks: 8 columns x every other row (32 rows); row chunks: 64 columns x 8 rows
    if (!make_map(&xc, x, BC, 8, 64, 2, kc, CU_TENSOR_MAP_L2_PROMOTION_NONE) ||
        !make_map(&lc, lam, 4 * BC, 8, 64, 2, kc, CU_TENSOR_MAP_L2_PROMOTION_NONE) ||
        !make_map(&xr, x, BC, 64, 8, 1, kc, CU_TENSOR_MAP_L2_PROMOTION_L2_128B) ||
        !make_map(&lr, lam, 4 * BC, 64, 8, 1, kc, CU_TENSOR_MAP_L2_PROMOTION_L2_128B))
        return GSPN_ERR_UNSUPPORTED;
    char* w = static_cast<char*>(ws);
    C64Args a;
    a.err = reinterpret_cast<int*>(w);
    a.wtab = reinterpret_cast<const float4*>(w + kWsAlign);
    a.out = static_cast<__nv_bfloat16*>(out);
    a.B = p.g.B;
    a.C = p.g.C;
    a.seg = S / p.g.groups;
    a.units = (int)(p.planes / kc);
    const int nw = p.g.B * 2 * S * S;
    c64_weights_kernel<__nv_bfloat16><<<(nw + 255) / 256, 256, 0, s>>>(
        static_cast<const __nv_bfloat16*>(logits), const_cast<float4*>(a.wtab), a.err, p.g.B);
    if (cudaGetLastError() != cudaSuccess) return GSPN_ERR_CUDA;
    const bool local = p.g.groups > 1;
    if (kc == 2)
        return local ? launch_c64<2, true>(dev, xc, lc, xr, lr, a, s) : launch_c64<2, false>(dev, xc, lc, xr, lr, a, s);
    return local ? launch_c64<1, true>(dev, xc, lc, xr, lr, a, s) : launch_c64<1, false>(dev, xc, lc, xr, lr, a, s);
}

}  // namespace gspn
