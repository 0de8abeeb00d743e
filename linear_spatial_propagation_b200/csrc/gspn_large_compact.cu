// gspn_large_compact.cu -- GSPN forward and backward of channel-shared
// (compact) bf16 planes whose lines are 129..256 positions long: 256x256
// latents and the like, the planes "Parallel Sequence Modeling via Generalized
// Spatial Propagation Network" scales to (one-line summary: 16K generation)
// with the compact weights of "GSPN-2: Efficient Parallel Sequence Modeling"
// (Justification for Channel-Agnostic Propagation).
//
// One warp owns one plane and walks its lines; lane t holds positions 8t..8t+7
// of a line in registers, so the three-tap mix needs two shuffles per line and
// no exchange between warps.  A CTA runs 8 warps = 8 consecutive channels of
// one batch image; they share the image's tap weights, which stream through a
// shared ring (one bulk copy per chunk of lines, issued by the last warp to
// finish with a stage) from a table a pre-kernel forms once per image (Key
// design 1: sigmoids of the tap logits, normalised over the taps that exist).
// Two warps per scheduler leave each warp up to 255 registers.
//
// The four directions of a plane run one after another and merge by summing
// through fp32 planes in the workspace (the planes do not fit on chip):
// * column scans (left->right, right->left) first; their running sum is kept
//   column-major (acct[plane][col][row]), so the sum of a column line is 8
//   contiguous floats per lane;
// * the first row scan reads that sum transposed by a 4-D tensor copy into
//   shared memory, the others row-major (acc[plane][row][col]);
// * the last direction writes the bf16 output.
// x and lambda (and dout in the backward) arrive by tensor copies into a ring
// per warp: rows as 256 x 4 boxes, columns as 8-column boxes through a
// (column, row / 8, row % 8, plane) view, so that lane t's reads of rows
// 8t..8t+7 are free of bank conflicts.  The warp issues its own copies, a ring
// ahead.  Every wait is bounded; an expired one sets the error word (workspace
// offset 0), drains the copies in flight and leaves.
//
// Backward (GSPN-2 response, "Backward Benchmark": the adjoint runs the same
// scan backwards with the transposed taps).  A first pass runs the forward
// and stores every direction's states h_i in scan order; the adjoint pass then
// walks each direction's lines from the last to the first:
//   a_i = dout_i + W_{i+1}^T a_{i+1}, i.e. a_i[j] = dout_i[j] + (1 - w0 - w2)(i+1, j) a[j]
//         + w0(i+1, j+1) a[j+1] + w2(i+1, j-1) a[j-1]   (no carry into a line
//         whose successor starts a local group),
//   dlambda_i = x_i a_i,  dx += lambda_i a_i  (merged over the directions as above),
//   E_k = a_i (h_{i-1}[j+k-1] - m_i[j]) for k = 0, 2, m_i the mix line i reads,
// summed over the channels; a last kernel forms dlogit_k = w_k (1 - s_k) E_k
// and dlogit_1 = -(1 - s_1)(w_0 E_0 + w_2 E_2) (the sigmoid and normalisation
// chain; sum_k w_k E_k = 0).
#include <cstring>
#include <type_traits>

#include "gspn_large_compact.h"
#include "gspn_lane.cuh"
#include "gspn_tma.cuh"

namespace gspn {

namespace {

using lane::FULL;

// order this thread's generic-proxy global-memory writes before later
// async-proxy (tensor copy) reads of the same memory
__device__ __forceinline__ void fence_proxy_async_global() { asm volatile("fence.proxy.async.global;" ::: "memory"); }
// four fp32 additions at the destination (16-byte aligned)
__device__ __forceinline__ void red_add4(float* p, float a, float b, float c, float d) {
    asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(a), "f"(b), "f"(c), "f"(d) : "memory");
}

constexpr int NCW = 8;                    // consumer warps (planes in flight per CTA)
constexpr int THREADS = NCW * 32;
constexpr int P = 8;                      // positions per lane
constexpr int LMAX = 256;                 // longest line
// data ring per warp: forward 3 stages of 8 KB (rows: x, lambda 2 KB each,
// column sums 4 KB; columns: x, lambda 4 KB each); adjoint 2 stages of 12 KB
// (dout as well)
template <bool ADJ>
struct Ring {
    static constexpr int NST = ADJ ? 2 : 3;
    static constexpr int STAGE = ADJ ? 12288 : 8192;
};
constexpr int RING = 3 * 8192;            // bytes per warp, both rings
constexpr int NTS = 4;                    // tap stages (4 lines each)
constexpr int TLINE = 2048;               // taps of one line: 256 positions x (w0, w2)
constexpr int TSTAGE = 4 * TLINE;
constexpr int OFF_T = NCW * RING;
constexpr int OFF_BAR = OFF_T + NTS * TSTAGE;
constexpr int NBAR = NCW * 3 + NTS + 1;
constexpr int OFF_CNT = OFF_BAR + NBAR * 8;          // per tap stage: warps done with it
constexpr int SMEM_BYTES = OFF_CNT + NTS * 4 + 128;  // + alignment slack
static_assert(Ring<true>::NST * Ring<true>::STAGE == RING && Ring<false>::NST * Ring<false>::STAGE == RING, "");

// k-th direction in processing order (columns first): dir | slot << 2 | in << 4 | out << 6
// in:  0 nothing (first direction), 1 column sums row by row (acct, direct loads),
//      2 column sums transposed (acct, tensor copy), 3 row sums (acc, direct loads)
// out: 0 column sums (acct), 1 row sums (acc), 2 the bf16 output (forward: out;
//      adjoint: dx), 3 the direction's states in scan order (backward's first pass)
struct LcArgs {
    const float4* taps;   // [slot][b][LMAX lines][4][32]: (-w0, -w0', w2, w2') of positions 8t+2q, 8t+2q+1
    float* acc;           // [plane][H][W]
    float* acct;          // [plane][W][H]
    __nv_bfloat16* out;   // forward: out; adjoint: dx
    float* hst;           // backward: [slot][plane][LMAX lines][LMAX] states
    float* esum;          // backward: [slot][b][LMAX lines][LMAX][2] tap values summed over channels
    __nv_bfloat16* dlam;  // backward: [slot][B][C][H][W]
    int* err;
    int B, C, H, W, D;
    int planes;           // B * C
    int kinfo[4];
    int groups;           // B * C / 8
    int segr, segc;       // local group lengths of row and column scans
    uint64_t limit;       // bound of every wait on data, a stage or another warp (ns)
    int stall;            // test hook: consumer warp 0 of CTA 0 first waits on a barrier nothing completes
};

__device__ __forceinline__ int kinfo_of(const LcArgs& a, int k) {
    return k == 0 ? a.kinfo[0] : k == 1 ? a.kinfo[1] : k == 2 ? a.kinfo[2] : a.kinfo[3];
}

// The taps table: one thread per (slot, image, line, quad q, lane t) writes the
// normalised (w0, w2) of positions 8t+2q and 8t+2q+1 of that line in scan
// order, w0 negated; positions beyond the line are zero.  Also clears the
// error word and (backward) the channel sums of the tap values.
__global__ void __launch_bounds__(256) lc_taps_kernel(const __nv_bfloat16* __restrict__ logits,
                                                      float4* __restrict__ taps, int* err, float* esum,
                                                      const Launch g) {
    const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx == 0) *err = 0;
    if (idx >= (int64_t)g.D * g.B * LMAX * 128) return;
    const int t = (int)(idx & 31), q = (int)((idx >> 5) & 3);
    const int i = (int)((idx >> 7) % LMAX);
    const int sb = (int)(idx / (128 * LMAX));  // slot * B + b
    if (esum)
        *reinterpret_cast<float4*>(esum + (((size_t)sb * LMAX + i) * LMAX + 8 * t + 2 * q) * 2) =
            make_float4(0.f, 0.f, 0.f, 0.f);
    const int slot = sb / g.B;
    const int d = dir_of(g, slot);
    const int L = scan_len(d, g.H, g.W), N = line_len(d, g.H, g.W);
    if (i >= L) return;
    const Walk wk = walk_of(d, g.H, g.W);
    const int HW = g.H * g.W;
    const __nv_bfloat16* const lg = logits + (size_t)sb * 3 * HW;
    float w[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int u = 0; u < 2; ++u) {
        const int j = 8 * t + 2 * q + u;
        if (j >= N) continue;
        const int pix = wk.o + i * wk.si + j * wk.sj;
        const float s0 = j > 0 ? sigmoidf(load_elt(lg, pix)) : 0.f;
        const float s1 = sigmoidf(load_elt(lg, HW + pix));
        const float s2 = j < N - 1 ? sigmoidf(load_elt(lg, 2 * HW + pix)) : 0.f;
        const float r = 1.f / (s0 + s1 + s2);
        w[u] = -s0 * r;
        w[2 + u] = s2 * r;
    }
    taps[idx] = make_float4(w[0], w[1], w[2], w[3]);
}

__device__ __forceinline__ float comp(const float4& v, int i) { return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w; }
__device__ __forceinline__ uint32_t swap_halves(uint32_t w) { return __byte_perm(w, 0, 0x1032); }

// The body of both scan kernels.  ADJ = false: the forward (out modes 0..3);
// ADJ = true: the adjoint pass of the backward, walking each direction's lines
// from the last to the first.
template <bool ADJ>
__device__ __forceinline__ void lc_body(const CUtensorMap& tm_xr, const CUtensorMap& tm_lr, const CUtensorMap& tm_gr,
                                        const CUtensorMap& tm_xc, const CUtensorMap& tm_lc, const CUtensorMap& tm_gc,
                                        const CUtensorMap& tm_at, const LcArgs& a) {
    constexpr int NST = Ring<ADJ>::NST, STAGE = Ring<ADJ>::STAGE;
    // stage layout: rows x | lambda | (dout) | column sums; columns x | lambda | (dout)
    constexpr int R_L = 2048, R_G = 4096, R_A = ADJ ? 6144 : 4096;
    constexpr int C_L = 4096, C_G = 8192;
    extern __shared__ __align__(128) unsigned char smem_raw[];
    unsigned char* const smem = smem_raw + ((128u - (tma::smem_u32(smem_raw) & 127u)) & 127u);
    const uint32_t sbase = tma::smem_u32(smem);
    const int warp = threadIdx.x >> 5, t = threadIdx.x & 31;
    const uint32_t full0 = sbase + OFF_BAR;            // full[w][s]: a warp's data stage has landed
    const uint32_t tfull0 = full0 + 8 * NCW * NST;      // tfull[s]: a tap stage has landed
    const uint32_t never = tfull0 + 8 * NTS;            // stall-test barrier: nothing completes it
    int* const tcount = reinterpret_cast<int*>(smem + OFF_CNT);
    // The walk over a direction's lines: ascending scan order in the forward,
    // descending in the adjoint.  `desc` is true when the walk goes down the
    // image (bottom->top rows, right->left columns).
    auto walk_desc = [&](int d) { return (d == B2T || d == R2L) != ADJ; };
    auto lines_of = [&](int d) { return d < 2 ? a.H : a.W; };
    // The taps stream in quads of 4 lines; every warp walks the same sequence
    // (group, direction index, quad).
    struct Cursor {
        int g, k, qd;
    };
    auto advance = [&](Cursor& c) {
        if (++c.qd == lines_of(kinfo_of(a, c.k) & 3) / 4) {
            c.qd = 0;
            if (++c.k == a.D) {
                c.k = 0;
                c.g += gridDim.x;
            }
        }
    };
    // one bulk copy of the taps of quad c into tap stage ts: scan lines 4qd ..
    // 4qd+3 (forward) or L-4-4qd .. L-1-4qd (adjoint)
    auto issue_taps = [&](const Cursor& c, int ts) {
        const int info = kinfo_of(a, c.k);
        const int slot = (info >> 2) & 3;
        const int first = ADJ ? lines_of(info & 3) - 4 - 4 * c.qd : 4 * c.qd;
        const int b = (8 * c.g) / a.C;
        const unsigned char* src = reinterpret_cast<const unsigned char*>(a.taps) +
                                   ((size_t)(slot * a.B + b) * LMAX + (size_t)first) * TLINE;
        tma::mbar_expect_tx(tfull0 + 8 * ts, TSTAGE);
        tma::load_1d(sbase + OFF_T + ts * TSTAGE, src, TSTAGE, tfull0 + 8 * ts);
    };
    if (threadIdx.x == 0) {
        for (int i = 0; i < NCW * NST; ++i) tma::mbar_init(full0 + 8 * i, 1);
        for (int s = 0; s < NTS; ++s) {
            tma::mbar_init(tfull0 + 8 * s, 1);
            tcount[s] = 0;
        }
        tma::mbar_init(never, 1);
        tma::fence_barrier_init();
    }
    if (threadIdx.x == 32) {
        tma::prefetch_map(&tm_xr);
        tma::prefetch_map(&tm_lr);
        if (ADJ) tma::prefetch_map(&tm_gr);
        if ((a.kinfo[0] & 3) >= 2) {  // the column maps exist only with a column direction (processed first)
            tma::prefetch_map(&tm_xc);
            tma::prefetch_map(&tm_lc);
            if (ADJ) tma::prefetch_map(&tm_gc);
            tma::prefetch_map(&tm_at);
        }
    }
    __syncthreads();
    // lane 0: the taps quad NTS ahead of this warp (a stage's refill), and per
    // tap stage the last quad this warp issued into it (-1: none)
    Cursor tnext{(int)blockIdx.x, 0, 0};
    int tlast[NTS];
#pragma unroll
    for (int s = 0; s < NTS; ++s) tlast[s] = -1;
    if (threadIdx.x == 0) {
#pragma unroll
        for (int s = 0; s < NTS; ++s) {
            if (tnext.g < a.groups) {
                issue_taps(tnext, s);
                tlast[s] = s;
                advance(tnext);
            }
        }
    } else {
        for (int s = 0; s < NTS && tnext.g < a.groups; ++s) advance(tnext);
    }

    // ---------------- consumer warps: one plane each ----------------
    unsigned char* const ring = smem + warp * RING;
    const uint32_t ringa = sbase + warp * RING;
    const uint32_t fullw = full0 + 8 * warp * NST;
    int n = 0;  // data chunks consumed
    int m = 0;  // taps quads consumed
    // lane 0: the next data chunk to issue
    int issued = 0, ig = blockIdx.x, ik = 0, ich = 0;
    auto nch_of = [&](int k) { return (kinfo_of(a, k) & 3) < 2 ? a.H / 4 : a.W / 8; };
    auto issue_one = [&]() {
        const int info = kinfo_of(a, ik);
        const int d = info & 3, slot = (info >> 2) & 3, in = (info >> 4) & 3;
        const int s = issued % NST;
        const uint32_t bar = fullw + 8 * s, dst = ringa + s * STAGE;
        const int pl = 8 * ig + warp;
        const int b = (8 * ig) / a.C, c = pl - b * a.C;
        const int lpl = (slot * a.B + b) * a.C + c;
        if (d < 2) {
            const int y0 = walk_desc(d) ? a.H - 4 - 4 * ich : 4 * ich;
            tma::mbar_expect_tx(bar, (ADJ ? 6144u : 4096u) + (in == 2 ? 4096u : 0u));
            tma::load_3d(dst, &tm_xr, 0, y0, pl, bar);
            tma::load_3d(dst + R_L, &tm_lr, 0, y0, lpl, bar);
            if (ADJ) tma::load_3d(dst + R_G, &tm_gr, 0, y0, pl, bar);
            if (in == 2) tma::load_4d(dst + R_A, &tm_at, y0, 0, 0, pl, bar);
        } else {
            const int x0 = walk_desc(d) ? a.W - 8 - 8 * ich : 8 * ich;
            tma::mbar_expect_tx(bar, ADJ ? 12288u : 8192u);
            tma::load_4d(dst, &tm_xc, x0, 0, 0, pl, bar);
            tma::load_4d(dst + C_L, &tm_lc, x0, 0, 0, lpl, bar);
            if (ADJ) tma::load_4d(dst + C_G, &tm_gc, x0, 0, 0, pl, bar);
        }
        ++issued;
        if (++ich == nch_of(ik)) {
            ich = 0;
            if (++ik == a.D) {
                ik = 0;
                ig += gridDim.x;
            }
        }
    };
    // Keep NST chunks in flight.  A chunk of a direction that reads the column
    // sums by tensor copy waits until this warp has finished writing them.
    auto issue_more = [&](int g, int k) {
        if (t == 0) {
            while (issued < n + NST && ig < a.groups) {
                if (((kinfo_of(a, ik) >> 4) & 3) == 2 && (ig != g || ik != k)) break;
                issue_one();
            }
        }
        __syncwarp();
    };
    auto fail = [&]() {
        if (t == 0) {
            atomicExch(a.err, 1);
            // the copies this warp issued land before the CTA can leave
            for (int mm = n; mm < issued; ++mm)
                tma::mbar_wait(fullw + 8 * (mm % NST), (mm / NST) & 1, 100000000ull);
#pragma unroll
            for (int s = 0; s < NTS; ++s)
                if (tlast[s] >= 0) tma::mbar_wait(tfull0 + 8 * s, (tlast[s] / NTS) & 1, 100000000ull);
        }
        __syncwarp();
    };

    // One direction of plane 8g + warp: walk steps k = 0 .. L-1 (scan line k in
    // the forward, L-1-k in the adjoint).
    auto run_dir = [&](auto rows_c, auto in_c, auto out_c, int g, int kdir) -> bool {
        constexpr bool ROWS = decltype(rows_c)::value;
        constexpr int IN = decltype(in_c)::value, OUT = decltype(out_c)::value;
        const int info = kinfo_of(a, kdir);
        const int d = info & 3, slot = (info >> 2) & 3;
        const bool desc = walk_desc(d);
        const int L = ROWS ? a.H : a.W, N = ROWS ? a.W : a.H;
        const int seg = ROWS ? a.segr : a.segc;
        const size_t pl = (size_t)(8 * g + warp);
        const bool act = 8 * t < N;  // this lane's positions lie on the line
        float* const accp = a.acc + pl * a.H * a.W;
        float* const actp = a.acct + pl * a.W * a.H;
        __nv_bfloat16* const outp = a.out + pl * a.H * a.W;
        // element offset of position 8t of the line at walk step k: row-major for
        // row lines, column-major for column lines
        auto line_off = [&](int k) -> size_t { return (size_t)(desc ? L - 1 - k : k) * N + 8 * t; };
        const float* const sump = IN == 1 ? actp : accp;
        float4 ar[4][2];  // IN 1, 3: the sums of the lines at walk steps k .. k+3, by k % 4
        if constexpr (IN == 1 || IN == 3) {
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                ar[r][0] = ar[r][1] = make_float4(0.f, 0.f, 0.f, 0.f);
                if (act && r < L) {
                    const float4* src = reinterpret_cast<const float4*>(sump + line_off(r));
                    ar[r][0] = src[0];
                    ar[r][1] = src[1];
                }
            }
        }
        // backward: this direction's states (scan order), the channel sums of the
        // tap values, dlambda
        const size_t sb = (size_t)slot * a.B + (8 * g) / a.C;
        float* const hstp = a.hst + ((size_t)slot * a.planes + pl) * LMAX * LMAX + 8 * t;
        [[maybe_unused]] float* const esp = a.esum + sb * LMAX * LMAX * 2 + 16 * t;
        __nv_bfloat16* const dlp = a.dlam + ((size_t)slot * a.planes + pl) * a.H * a.W;
        float h[P];  // forward: the state; adjoint: a
#pragma unroll
        for (int p = 0; p < P; ++p) h[p] = 0.f;
        // adjoint: the states of line i-1 for walk steps k, k+1 (by k % 2), and
        // the taps of line i+1 (the previous step's line)
        [[maybe_unused]] float hr_[2][P];
        [[maybe_unused]] float4 TN[4];
        if constexpr (ADJ) {
#pragma unroll
            for (int r = 0; r < 2; ++r) {
#pragma unroll
                for (int p = 0; p < P; ++p) hr_[r][p] = 0.f;
                const int li = L - 2 - r;
                if (act && li >= 0) {
                    const float4* src = reinterpret_cast<const float4*>(hstp + (size_t)li * LMAX);
                    const float4 u = src[0], v = src[1];
                    hr_[r][0] = u.x; hr_[r][1] = u.y; hr_[r][2] = u.z; hr_[r][3] = u.w;
                    hr_[r][4] = v.x; hr_[r][5] = v.y; hr_[r][6] = v.z; hr_[r][7] = v.w;
                }
            }
#pragma unroll
            for (int q = 0; q < 4; ++q) TN[q] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
        // i % seg of the line at the current walk step, kept by counting
        int gpos = ADJ ? seg - 1 : 0;
        int nt = 0;                      // the data chunk being read
        const unsigned char* st = ring;  // its stage
        uint4 X[ROWS ? 4 : 1], Lm[ROWS ? 4 : 1];
        [[maybe_unused]] uint4 G[ROWS && ADJ ? 4 : 1];  // rows: line e, positions 8t..8t+7
        uint2 Xh[ROWS ? 1 : P], Lh[ROWS ? 1 : P];
        [[maybe_unused]] uint2 Gh[!ROWS && ADJ ? P : 1];  // columns: row 8t+p, the quad's 4 lines
        uint2 DL[!ROWS && ADJ ? P : 1];  // adjoint, columns: dlambda of the quad's 4 lines, row 8t+p, walk order
        float4 A[IN == 2 ? P : 1];
        // the stage's reads are done: hand it back to this warp's next copies
        auto release = [&]() {
            tma::fence_proxy_async();  // these reads come before the stage's refill
            __syncwarp();
            ++n;
            issue_more(g, kdir);
        };
        // columns: the quad's lines are the first or second 4 columns of the
        // box in walk order (the 8-byte piece at the other end, reversed, when
        // the walk goes right->left)
        auto read_half = [&](int hh) {
#pragma unroll
            for (int p = 0; p < P; ++p) {
                const int o = (p * 32 + t) * 16 + 8 * (desc ? 1 - hh : hh);
                const uint2 xv = *reinterpret_cast<const uint2*>(st + o);
                const uint2 lv = *reinterpret_cast<const uint2*>(st + C_L + o);
                Xh[p] = desc ? make_uint2(swap_halves(xv.y), swap_halves(xv.x)) : xv;
                Lh[p] = desc ? make_uint2(swap_halves(lv.y), swap_halves(lv.x)) : lv;
                if constexpr (ADJ) {
                    const uint2 gv = *reinterpret_cast<const uint2*>(st + C_G + o);
                    Gh[p] = desc ? make_uint2(swap_halves(gv.y), swap_halves(gv.x)) : gv;
                }
            }
        };
        const int nq = L / 4;
        for (int qd = 0; qd < nq; ++qd) {
            // data: one row chunk per quad, one column chunk per two quads
            if (ROWS || (qd & 1) == 0) {
                nt = n;
                const int s = nt % NST;
                if (!__all_sync(FULL, tma::mbar_wait(fullw + 8 * s, (nt / NST) & 1, a.limit))) return false;
                st = ring + s * STAGE;
                if constexpr (ROWS) {
                    // walk step e of the chunk is stage row e, or 3-e when the walk goes up
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int r = desc ? 3 - e : e;
                        X[e] = lane::lds128(st + r * 512 + t * 16);
                        Lm[e] = lane::lds128(st + R_L + r * 512 + t * 16);
                        if constexpr (ADJ) G[e] = lane::lds128(st + R_G + r * 512 + t * 16);
                    }
                    if constexpr (IN == 2) {
                        // column 8t+p of the chunk's 4 rows
#pragma unroll
                        for (int p = 0; p < P; ++p) {
                            const float4 v = lane::lds128f(st + R_A + (p * 32 + t) * 16);
                            A[p] = desc ? make_float4(v.w, v.z, v.y, v.x) : v;
                        }
                    }
                    release();
                } else {
                    read_half(0);
                }
            } else {
                read_half(1);
                release();
            }
            const int mt = m++;
            const int ts = mt % NTS;
            if (!__all_sync(FULL, tma::mbar_wait(tfull0 + 8 * ts, (mt / NTS) & 1, a.limit))) return false;
            const unsigned char* tp = smem + OFF_T + ts * TSTAGE + t * 16;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int k = 4 * qd + e;          // walk step
                const int i = ADJ ? L - 1 - k : k;  // scan line
                float4 T[4];  // taps of line i: the quad's line e (forward) or 3-e (adjoint)
#pragma unroll
                for (int q = 0; q < 4; ++q) T[q] = lane::lds128f(tp + (ADJ ? 3 - e : e) * TLINE + q * 512);
                float v[P];  // what this direction adds to the merged sum at the line
                if constexpr (!ADJ) {
                    if (gpos == 0) {
#pragma unroll
                        for (int p = 0; p < P; ++p) h[p] = 0.f;  // a scan or local group starts: h_{-1} = 0
                    }
                    gpos = gpos + 1 == seg ? 0 : gpos + 1;
                    float base[P];
#pragma unroll
                    for (int p = 0; p < P; ++p) {
                        if constexpr (ROWS)
                            base[p] = lane::fma_bf(p & 1, lane::word_of(Lm[e], p >> 1), lane::word_of(X[e], p >> 1), h[p]);
                        else
                            base[p] = lane::fma_bf(e & 1, (e & 2) ? Lh[p].y : Lh[p].x, (e & 2) ? Xh[p].y : Xh[p].x, h[p]);
                    }
                    // neighbours of the previous line; the rotation brings lane 31's last
                    // position to lane 0 and lane 0's first to lane 31, where w0 = 0 and w2 = 0
                    const float hl = __shfl_sync(FULL, h[P - 1], (t + 31) & 31);
                    const float hr = __shfl_sync(FULL, h[0], (t + 1) & 31);
                    float dd[P + 1];  // dd[p] = h[p] - h[p-1]
                    dd[0] = h[0] - hl;
#pragma unroll
                    for (int p = 1; p < P; ++p) dd[p] = h[p] - h[p - 1];
                    dd[P] = hr - h[P - 1];
                    // h' = lambda x + h + w0 (h[j-1] - h) + w2 (h[j+1] - h)
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        h[2 * q] = fmaf(T[q].x, dd[2 * q], fmaf(T[q].z, dd[2 * q + 1], base[2 * q]));
                        h[2 * q + 1] = fmaf(T[q].y, dd[2 * q + 1], fmaf(T[q].w, dd[2 * q + 2], base[2 * q + 1]));
                    }
#pragma unroll
                    for (int p = 0; p < P; ++p) v[p] = h[p];
                } else {
                    // the line's x, lambda and dout at positions 8t..8t+7
                    float xs[P], ls[P], gs[P];
#pragma unroll
                    for (int p = 0; p < P; ++p) {
                        uint32_t xw, lw, gw;
                        int half;
                        if constexpr (ROWS) {
                            xw = lane::word_of(X[e], p >> 1);
                            lw = lane::word_of(Lm[e], p >> 1);
                            gw = lane::word_of(G[e], p >> 1);
                            half = p & 1;
                        } else {
                            xw = (e & 2) ? Xh[p].y : Xh[p].x;
                            lw = (e & 2) ? Lh[p].y : Lh[p].x;
                            gw = (e & 2) ? Gh[p].y : Gh[p].x;
                            half = e & 1;
                        }
                        xs[p] = __uint_as_float(half ? (xw & 0xffff0000u) : (xw << 16));
                        ls[p] = __uint_as_float(half ? (lw & 0xffff0000u) : (lw << 16));
                        gs[p] = __uint_as_float(half ? (gw & 0xffff0000u) : (gw << 16));
                    }
                    // line i reads line i-1 (carry_out) unless it starts a group; line
                    // i+1 read line i (carry_in) unless it starts one
                    const bool carry_out = gpos != 0;
                    const bool carry_in = k > 0 && gpos != seg - 1;
                    gpos = gpos == 0 ? seg - 1 : gpos - 1;
                    // a_i = dout + a - w0 a - w2 a + (w0 a)[j+1] + (w2 a)[j-1], taps of line
                    // i+1; the shuffles rotate (lane 31 takes w0 a of position 0, lane 0
                    // w2 a of position 255: both taps are zero there)
                    float p0[P], p2[P];
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        p0[2 * q] = -TN[q].x * h[2 * q];
                        p0[2 * q + 1] = -TN[q].y * h[2 * q + 1];
                        p2[2 * q] = TN[q].z * h[2 * q];
                        p2[2 * q + 1] = TN[q].w * h[2 * q + 1];
                    }
                    const float p0r = __shfl_sync(FULL, p0[0], (t + 1) & 31);
                    const float p2l = __shfl_sync(FULL, p2[P - 1], (t + 31) & 31);
#pragma unroll
                    for (int p = 0; p < P; ++p) {
                        const float right = p < P - 1 ? p0[p + 1] : p0r;
                        const float left = p > 0 ? p2[p - 1] : p2l;
                        h[p] = carry_in ? gs[p] + ((h[p] - p0[p] - p2[p]) + (right + left)) : gs[p];
                        v[p] = ls[p] * h[p];  // this direction's share of dx
                    }
                    // tap values of line i, from the states of line i-1 and the mix m it reads
                    {
                        const float* hp = hr_[e & 1];
                        const float hpl = __shfl_sync(FULL, hp[P - 1], (t + 31) & 31);
                        const float hpr = __shfl_sync(FULL, hp[0], (t + 1) & 31);
                        if (carry_out && act) {
                            float ev[2 * P];
#pragma unroll
                            for (int q = 0; q < 4; ++q) {
#pragma unroll
                                for (int u = 0; u < 2; ++u) {
                                    const int p = 2 * q + u;
                                    const float nw0 = u ? T[q].y : T[q].x, w2 = u ? T[q].w : T[q].z;
                                    const float hm = p > 0 ? hp[p - 1] : hpl, hq = p < P - 1 ? hp[p + 1] : hpr;
                                    const float mix = fmaf(w2, hq - hp[p], fmaf(-nw0, hm - hp[p], hp[p]));
                                    ev[2 * p] = h[p] * (hm - mix);
                                    ev[2 * p + 1] = h[p] * (hq - mix);
                                }
                            }
                            float* dst = esp + (size_t)i * LMAX * 2;
#pragma unroll
                            for (int r = 0; r < 4; ++r)
                                red_add4(dst + 4 * r, ev[4 * r], ev[4 * r + 1], ev[4 * r + 2], ev[4 * r + 3]);
                        }
                    }
                    // dlambda = x a: rows straight to memory, columns a quad at a time
                    if constexpr (ROWS) {
                        if (act) {
                            const uint4 w = make_uint4(lane::pack_bf2(xs[0] * h[0], xs[1] * h[1]),
                                                       lane::pack_bf2(xs[2] * h[2], xs[3] * h[3]),
                                                       lane::pack_bf2(xs[4] * h[4], xs[5] * h[5]),
                                                       lane::pack_bf2(xs[6] * h[6], xs[7] * h[7]));
                            *reinterpret_cast<uint4*>(dlp + line_off(k)) = w;
                        }
                    } else {
#pragma unroll
                        for (int p = 0; p < P; ++p) {
                            const uint32_t bits = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(xs[p] * h[p]));
                            uint32_t& word = (e & 2) ? DL[p].y : DL[p].x;
                            word = (e & 1) ? (word | (bits << 16)) : bits;
                        }
                    }
                    // the taps of this line serve the next step as line i+1; the states
                    // slot of this step takes line i-3 (the step after next reads it)
#pragma unroll
                    for (int q = 0; q < 4; ++q) TN[q] = T[q];
                    {
                        const int li = i - 3;
                        if (act && li >= 0) {
                            const float4* src = reinterpret_cast<const float4*>(hstp + (size_t)li * LMAX);
                            const float4 u = src[0], w = src[1];
                            float* hw = hr_[e & 1];
                            hw[0] = u.x; hw[1] = u.y; hw[2] = u.z; hw[3] = u.w;
                            hw[4] = w.x; hw[5] = w.y; hw[6] = w.z; hw[7] = w.w;
                        }
                    }
                }
#pragma unroll
                for (int p = 0; p < P; ++p) {
                    float sprev = 0.f;
                    if constexpr (IN == 1 || IN == 3) sprev = comp(ar[e][p >> 2], p & 3);
                    if constexpr (IN == 2) sprev = comp(A[p], e);
                    v[p] += sprev;
                }
                if (act) {
                    const size_t o = line_off(k);
                    if constexpr (OUT == 2) {
                        const uint4 w = make_uint4(lane::pack_bf2(v[0], v[1]), lane::pack_bf2(v[2], v[3]),
                                                   lane::pack_bf2(v[4], v[5]), lane::pack_bf2(v[6], v[7]));
                        *reinterpret_cast<uint4*>(outp + o) = w;
                    } else if constexpr (OUT == 3) {
                        float4* dst = reinterpret_cast<float4*>(hstp + (size_t)i * LMAX);
                        dst[0] = make_float4(v[0], v[1], v[2], v[3]);
                        dst[1] = make_float4(v[4], v[5], v[6], v[7]);
                    } else {
                        float4* dst = reinterpret_cast<float4*>((OUT == 0 ? actp : accp) + o);
                        dst[0] = make_float4(v[0], v[1], v[2], v[3]);
                        dst[1] = make_float4(v[4], v[5], v[6], v[7]);
                    }
                }
                if constexpr (IN == 1 || IN == 3) {
                    if (act && k + 4 < L) {
                        const float4* src = reinterpret_cast<const float4*>(sump + line_off(k + 4));
                        ar[e][0] = src[0];
                        ar[e][1] = src[1];
                    }
                }
            }
            if constexpr (ADJ && !ROWS) {
                // the quad's 4 columns of rows 8t..8t+7: one 8-byte store per row, in
                // column order
                if (act) {
                    const int colbase = desc ? L - 4 - 4 * qd : 4 * qd;
#pragma unroll
                    for (int p = 0; p < P; ++p) {
                        const uint2 w = desc ? make_uint2(swap_halves(DL[p].y), swap_halves(DL[p].x)) : DL[p];
                        *reinterpret_cast<uint2*>(dlp + (size_t)(8 * t + p) * a.W + colbase) = w;
                    }
                }
            }
            // This warp is done with the tap stage; the last of the 8 warps refills
            // it with the quad NTS ahead.  Each lane orders its reads before the
            // copy (proxy fence); the fences around the counter order the warps.
            tma::fence_proxy_async();
            __syncwarp();
            if (t == 0) {
                __threadfence_block();
                if (atomicAdd(tcount + ts, 1) == NCW - 1) {
                    __threadfence_block();
                    tcount[ts] = 0;
                    if (tnext.g < a.groups) {
                        issue_taps(tnext, ts);
#pragma unroll
                        for (int s = 0; s < NTS; ++s)
                            if (s == ts) tlast[s] = mt + NTS;
                    }
                }
                advance(tnext);
            }
            __syncwarp();
        }
        return true;
    };

    using tru = std::true_type;
    using fal = std::false_type;
    using i0 = std::integral_constant<int, 0>;
    using i1 = std::integral_constant<int, 1>;
    using i2 = std::integral_constant<int, 2>;
    using i3 = std::integral_constant<int, 3>;
    bool ok = true;
    if (a.stall && blockIdx.x == 0 && warp == 0) {
        // test hook: nothing completes `never`, so this wait can only run out
        ok = __all_sync(FULL, tma::mbar_wait(never, 0, a.limit));
    }
    if (ok) issue_more(blockIdx.x, 0);
    for (int g = blockIdx.x; ok && g < a.groups; g += gridDim.x) {
        for (int k = 0; ok && k < a.D; ++k) {
            const int info = kinfo_of(a, k);
            const int d = info & 3, in = (info >> 4) & 3, out = (info >> 6) & 3;
            if (in == 2) {
                // the column sums this warp stored (generic proxy) are read next by tensor copies
                fence_proxy_async_global();
                __syncwarp();
                issue_more(g, k);
            }
            if (!ADJ && out == 3)
                ok = d >= 2 ? run_dir(fal{}, i0{}, i3{}, g, k) : run_dir(tru{}, i0{}, i3{}, g, k);
            else if (d >= 2)
                ok = in == 0 ? run_dir(fal{}, i0{}, i0{}, g, k) : run_dir(fal{}, i1{}, i0{}, g, k);
            else if (in == 0)
                ok = out == 1 ? run_dir(tru{}, i0{}, i1{}, g, k) : run_dir(tru{}, i0{}, i2{}, g, k);
            else if (in == 2)
                ok = out == 1 ? run_dir(tru{}, i2{}, i1{}, g, k) : run_dir(tru{}, i2{}, i2{}, g, k);
            else
                ok = run_dir(tru{}, i3{}, i2{}, g, k);
        }
    }
    if (!ok) fail();
}

__global__ void __launch_bounds__(THREADS, 1)
    lc_fwd_kernel(const __grid_constant__ CUtensorMap tm_xr, const __grid_constant__ CUtensorMap tm_lr,
                  const __grid_constant__ CUtensorMap tm_xc, const __grid_constant__ CUtensorMap tm_lc,
                  const __grid_constant__ CUtensorMap tm_at, const LcArgs a) {
    lc_body<false>(tm_xr, tm_lr, tm_xr, tm_xc, tm_lc, tm_xc, tm_at, a);
}

__global__ void __launch_bounds__(THREADS, 1)
    lc_adj_kernel(const __grid_constant__ CUtensorMap tm_xr, const __grid_constant__ CUtensorMap tm_lr,
                  const __grid_constant__ CUtensorMap tm_gr, const __grid_constant__ CUtensorMap tm_xc,
                  const __grid_constant__ CUtensorMap tm_lc, const __grid_constant__ CUtensorMap tm_gc,
                  const __grid_constant__ CUtensorMap tm_at, const LcArgs a) {
    lc_body<true>(tm_xr, tm_lr, tm_gr, tm_xc, tm_lc, tm_gc, tm_at, a);
}

// dlogits of the channel-shared taps from the channel sums of the tap values:
// one thread per (slot, image, pixel).  With s_k the sigmoids of the valid taps
// and w_k = s_k / sum s: dlogit_0 = w_0 (1 - s_0) E_0, dlogit_2 = w_2 (1 - s_2) E_2,
// dlogit_1 = -(1 - s_1)(w_0 E_0 + w_2 E_2); invalid taps (w_k = 0) get 0.
__global__ void __launch_bounds__(256) lc_dlogits_kernel(const __nv_bfloat16* __restrict__ logits,
                                                         const float* __restrict__ esum,
                                                         __nv_bfloat16* __restrict__ dlogits, const Launch g) {
    const int HW = g.H * g.W;
    const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= (int64_t)g.D * g.B * HW) return;
    const int pix = (int)(idx % HW);
    const int sb = (int)(idx / HW);
    const int d = dir_of(g, sb / g.B);
    const int r = pix / g.W, c = pix % g.W;
    const int i = d == T2B ? r : d == B2T ? g.H - 1 - r : d == L2R ? c : g.W - 1 - c;
    const int j = d < 2 ? c : r;
    const int N = line_len(d, g.H, g.W);
    const __nv_bfloat16* const lg = logits + (size_t)sb * 3 * HW;
    const float s0 = j > 0 ? sigmoidf(load_elt(lg, pix)) : 0.f;
    const float s1 = sigmoidf(load_elt(lg, HW + pix));
    const float s2 = j < N - 1 ? sigmoidf(load_elt(lg, 2 * HW + pix)) : 0.f;
    const float rr = 1.f / (s0 + s1 + s2);
    const float w0 = s0 * rr, w2 = s2 * rr;
    const float2 e = *reinterpret_cast<const float2*>(esum + (((size_t)sb * LMAX + i) * LMAX + j) * 2);
    __nv_bfloat16* const out = dlogits + (size_t)sb * 3 * HW + pix;
    out[0] = __float2bfloat16_rn(w0 * (1.f - s0) * e.x);
    out[HW] = __float2bfloat16_rn(-(1.f - s1) * (w0 * e.x + w2 * e.y));
    out[2 * HW] = __float2bfloat16_rn(w2 * (1.f - s2) * e.y);
}

// ---- host side ----------------------------------------------------------------
// (column, row, plane) view of bf16 planes; boxes of 256 columns x 4 rows
bool map_rows(CUtensorMap* m, const void* base, int H, int W, uint64_t planes) {
    EncodeTiledFn fn = encode_tiled();
    if (!fn) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)W, (cuuint64_t)H, planes};
    const cuuint64_t strides[2] = {(cuuint64_t)W * 2, (cuuint64_t)H * W * 2};
    const cuuint32_t box[3] = {LMAX, 4, 1};
    const cuuint32_t es[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// (column, row / 8, row % 8, plane) view of bf16 planes; boxes of 8 columns x
// all rows, laid out [row % 8][row / 8][8 columns]
bool map_cols(CUtensorMap* m, const void* base, int H, int W, uint64_t planes) {
    EncodeTiledFn fn = encode_tiled();
    if (!fn) return false;
    const cuuint64_t dims[4] = {(cuuint64_t)W, (cuuint64_t)H / 8, 8, planes};
    const cuuint64_t strides[3] = {(cuuint64_t)W * 2 * 8, (cuuint64_t)W * 2, (cuuint64_t)H * W * 2};
    const cuuint32_t box[4] = {8, LMAX / 8, 8, 1};
    const cuuint32_t es[4] = {1, 1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// (row, column / 8, column % 8, plane) view of the column-major fp32 sums
// acct[plane][col][row]; boxes of 4 rows x all columns, laid out
// [column % 8][column / 8][4 rows]
bool map_sums_t(CUtensorMap* m, const void* base, int H, int W, uint64_t planes) {
    EncodeTiledFn fn = encode_tiled();
    if (!fn) return false;
    const cuuint64_t dims[4] = {(cuuint64_t)H, (cuuint64_t)W / 8, 8, planes};
    const cuuint64_t strides[3] = {(cuuint64_t)H * 4 * 8, (cuuint64_t)H * 4, (cuuint64_t)H * W * 4};
    const cuuint32_t box[4] = {4, LMAX / 8, 8, 1};
    const cuuint32_t es[4] = {1, 1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, const_cast<void*>(base), dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int row_dirs(const Problem& p) { return __builtin_popcount(p.d.dir_mask & 3u); }
int col_dirs(const Problem& p) { return __builtin_popcount(p.d.dir_mask & 12u); }

size_t taps_bytes(const Problem& p) { return align_up((size_t)p.g.D * p.g.B * LMAX * TLINE, kWsAlign); }
size_t sums_bytes(const Problem& p) { return align_up((size_t)p.planes * p.HW * sizeof(float), kWsAlign); }
size_t esum_bytes(const Problem& p) {
    return align_up((size_t)p.g.D * p.g.B * LMAX * LMAX * 2 * sizeof(float), kWsAlign);
}
size_t states_bytes(const Problem& p) {
    return align_up((size_t)p.g.D * p.planes * LMAX * LMAX * sizeof(float), kWsAlign);
}

// Common arguments; the merged sums (row sums with two row directions, column
// sums with any column direction) start at `sums` in the workspace.
LcArgs base_args(const Problem& p, char* ws, char* sums, void* out) {
    LcArgs a;
    std::memset(&a, 0, sizeof(a));
    a.err = reinterpret_cast<int*>(ws);
    a.taps = reinterpret_cast<const float4*>(ws + kWsAlign);
    if (row_dirs(p) == 2) {
        a.acc = reinterpret_cast<float*>(sums);
        sums += sums_bytes(p);
    }
    if (col_dirs(p)) a.acct = reinterpret_cast<float*>(sums);
    a.out = static_cast<__nv_bfloat16*>(out);
    a.B = p.g.B;
    a.C = p.g.C;
    a.H = p.g.H;
    a.W = p.g.W;
    a.D = p.g.D;
    a.planes = (int)p.planes;
    a.groups = (int)(p.planes / 8);
    a.segr = p.g.H / p.g.groups;
    a.segc = p.g.W / p.g.groups;
    const WaitCfg wc = wait_cfg();
    a.limit = wc.limit_ns;
    a.stall = wc.stall;
    // processing order: left->right, right->left, top->bottom, bottom->top (those enabled)
    const int order[4] = {L2R, R2L, T2B, B2T};
    int k = 0, prev = -1;
    for (int o = 0; o < 4; ++o) {
        const int d = order[o];
        if (!(p.d.dir_mask & (1u << d))) continue;
        const int slot = __builtin_popcount(p.d.dir_mask & ((1u << d) - 1u));
        const bool rows = d < 2;
        const int in = prev < 0 ? 0 : !rows ? 1 : prev >= 2 ? 2 : 3;
        const int outm = k == p.g.D - 1 ? 2 : rows ? 1 : 0;
        a.kinfo[k++] = d | slot << 2 | in << 4 | outm << 6;
        prev = d;
    }
    return a;
}

bool make_maps(const Problem& p, const void* x, const void* lam, const void* dout, const float* acct, CUtensorMap* xr,
               CUtensorMap* lr, CUtensorMap* gr, CUtensorMap* xc, CUtensorMap* lc, CUtensorMap* gc, CUtensorMap* at) {
    const uint64_t BC = (uint64_t)p.planes, DBC = (uint64_t)p.g.D * BC;
    const int H = p.g.H, W = p.g.W;
    std::memset(gr, 0, sizeof(*gr));
    std::memset(xc, 0, sizeof(*xc));
    std::memset(lc, 0, sizeof(*lc));
    std::memset(gc, 0, sizeof(*gc));
    std::memset(at, 0, sizeof(*at));
    if (!map_rows(xr, x, H, W, BC) || !map_rows(lr, lam, H, W, DBC)) return false;
    if (dout && !map_rows(gr, dout, H, W, BC)) return false;
    if (col_dirs(p)) {
        if (!map_cols(xc, x, H, W, BC) || !map_cols(lc, lam, H, W, DBC) || !map_sums_t(at, acct, H, W, BC))
            return false;
        if (dout && !map_cols(gc, dout, H, W, BC)) return false;
    }
    return true;
}

gspn_status launch_taps(const Problem& p, const void* logits, const LcArgs& a, float* esum, cudaStream_t s) {
    const int64_t nt = (int64_t)p.g.D * p.g.B * LMAX * 128;
    lc_taps_kernel<<<(unsigned)((nt + 255) / 256), 256, 0, s>>>(static_cast<const __nv_bfloat16*>(logits),
                                                                const_cast<float4*>(a.taps), a.err, esum, p.g);
    return cudaGetLastError() == cudaSuccess ? GSPN_OK : GSPN_ERR_CUDA;
}

gspn_status launch_fwd(const DeviceInfo& dev, const CUtensorMap& xr, const CUtensorMap& lr, const CUtensorMap& xc,
                       const CUtensorMap& lc, const CUtensorMap& at, const LcArgs& a, cudaStream_t s) {
    const void* fn = (const void*)lc_fwd_kernel;
    if (ensure_smem_attr(fn, SMEM_BYTES, 43) != cudaSuccess) return GSPN_ERR_CUDA;
    const int grid = a.groups < dev.sm_count ? a.groups : dev.sm_count;
    lc_fwd_kernel<<<grid, THREADS, SMEM_BYTES, s>>>(xr, lr, xc, lc, at, a);
    return cudaGetLastError() == cudaSuccess ? GSPN_OK : GSPN_ERR_CUDA;
}

}  // namespace

// Compact bf16 planes with lines of 129..256 positions (H, W multiples of 8, at
// most 256, one of them above 128), whole groups of 8 channels, and at least
// one row direction (the last direction processed writes the output row by row).
bool lc_eligible(const Problem& p) {
    const int H = p.g.H, W = p.g.W;
    return p.d.dtype == GSPN_BF16 && p.g.shared && (p.d.dir_mask & 3u) && H <= LMAX && W <= LMAX &&
           (H > 128 || W > 128) && H % 8 == 0 && W % 8 == 0 && p.g.C % 8 == 0 &&
           p.planes * p.g.D <= ((int64_t)1 << 28) && encode_tiled() != nullptr;
}

// error word, taps table, row sums (two row directions), column sums (any column direction)
size_t lc_fwd_workspace(const Problem& p) {
    return kWsAlign + taps_bytes(p) + (row_dirs(p) == 2 ? sums_bytes(p) : 0) + (col_dirs(p) ? sums_bytes(p) : 0);
}

gspn_status lc_fwd(const Problem& p, const DeviceInfo& dev, const void* x, const void* logits, const void* lam,
                   void* out, void* ws, cudaStream_t s) {
    char* w = static_cast<char*>(ws);
    const LcArgs a = base_args(p, w, w + kWsAlign + taps_bytes(p), out);
    CUtensorMap xr, lr, gr, xc, lc, gc, at;
    if (!make_maps(p, x, lam, nullptr, a.acct, &xr, &lr, &gr, &xc, &lc, &gc, &at)) return GSPN_ERR_UNSUPPORTED;
    const gspn_status st = launch_taps(p, logits, a, nullptr, s);
    if (st != GSPN_OK) return st;
    return launch_fwd(dev, xr, lr, xc, lc, at, a, s);
}

// error word, taps table, tap-value sums, states, then the dx sums as in the forward
size_t lc_bwd_workspace(const Problem& p) {
    return kWsAlign + taps_bytes(p) + esum_bytes(p) + states_bytes(p) + (row_dirs(p) == 2 ? sums_bytes(p) : 0) +
           (col_dirs(p) ? sums_bytes(p) : 0);
}

gspn_status lc_bwd(const Problem& p, const DeviceInfo& dev, const void* x, const void* logits, const void* lam,
                   const void* dout, void* dx, void* dlogits, void* dlam, void* ws, cudaStream_t s) {
    char* w = static_cast<char*>(ws);
    char* const esum = w + kWsAlign + taps_bytes(p);
    char* const hst = esum + esum_bytes(p);
    LcArgs a = base_args(p, w, hst + states_bytes(p), dx);
    a.hst = reinterpret_cast<float*>(hst);
    a.esum = reinterpret_cast<float*>(esum);
    a.dlam = static_cast<__nv_bfloat16*>(dlam);
    CUtensorMap xr, lr, gr, xc, lc, gc, at;
    if (!make_maps(p, x, lam, dout, a.acct, &xr, &lr, &gr, &xc, &lc, &gc, &at)) return GSPN_ERR_UNSUPPORTED;
    gspn_status st = launch_taps(p, logits, a, a.esum, s);
    if (st != GSPN_OK) return st;
    // 1. the forward of every direction, its states stored in scan order
    LcArgs f = a;
    for (int k = 0; k < a.D; ++k) f.kinfo[k] = (a.kinfo[k] & 15) | 3 << 6;
    st = launch_fwd(dev, xr, lr, xc, lc, at, f, s);
    if (st != GSPN_OK) return st;
    // 2. the adjoint: dlambda, dx (merged over the directions), tap-value sums
    const void* fn = (const void*)lc_adj_kernel;
    if (ensure_smem_attr(fn, SMEM_BYTES, 44) != cudaSuccess) return GSPN_ERR_CUDA;
    const int grid = a.groups < dev.sm_count ? a.groups : dev.sm_count;
    lc_adj_kernel<<<grid, THREADS, SMEM_BYTES, s>>>(xr, lr, gr, xc, lc, gc, at, a);
    if (cudaGetLastError() != cudaSuccess) return GSPN_ERR_CUDA;
    // 3. dlogits
    const int64_t n = (int64_t)p.g.D * p.g.B * p.HW;
    lc_dlogits_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(
        static_cast<const __nv_bfloat16*>(logits), a.esum, static_cast<__nv_bfloat16*>(dlogits), p.g);
    return cudaGetLastError() == cudaSuccess ? GSPN_OK : GSPN_ERR_CUDA;
}

}  // namespace gspn
