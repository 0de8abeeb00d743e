// gspn_generic.cu -- the generic GSPN kernels: any B, C, H, W, dtype, direction
// set, local-group count and weight mode.
//
// One warp owns one (b, c) plane.  For each enabled direction it walks the
// lines in scan order ("Parallel Sequence Modeling via Generalized Spatial
// Propagation Network", Key design 2: lines are sequential, the positions of
// a line are independent); lane l computes positions l, l+32, ... of the
// line.  The previous line lives in a per-warp shared-memory buffer with a
// zero halo at both ends, so tap k of position j reads buffer slot j+k.  The
// four directions are summed (the merge) into an fp32 plane accumulator that
// lives in shared memory when it fits and in the workspace otherwise; the
// plane is written once at the end.
//
// The tap weights are recomputed from the logits where they are used:
// s_k = sigmoid(logit_k) for the taps whose source lies in the line,
// w_k = s_k / sum of those s (Key design 1).
#include "gspn_internal.h"

namespace gspn {

namespace {

constexpr int kMaxWarps = 8;
constexpr int kSmemBudget = 200 * 1024;

struct FwdArgs {
    Launch g;
    const void* x;
    const void* logits;
    const void* lam;
    void* out;
    float* acc_ws;
    int acc_in_smem;
    int warps_per_cta;
    int lstride;  // floats per line buffer (N_max + 2)
};

template <typename T>
__global__ void __launch_bounds__(kMaxWarps * 32) generic_fwd_kernel(FwdArgs a) {
    extern __shared__ float smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int H = a.g.H, W = a.g.W, HW = H * W, B = a.g.B, C = a.g.C;
    const int64_t plane = (int64_t)blockIdx.x * a.warps_per_cta + warp;
    if (plane >= (int64_t)B * C) return;
    float* wsm = smem + (size_t)warp * (2 * a.lstride + (a.acc_in_smem ? HW : 0));
    float* acc = a.acc_in_smem ? wsm + 2 * a.lstride : a.acc_ws + plane * HW;
    const int64_t b = plane / C, c = plane % C, cw = a.g.shared ? 0 : c;
    const int Cw = a.g.shared ? 1 : C;
    const T* x = static_cast<const T*>(a.x) + plane * HW;

    for (int slot = 0; slot < a.g.D; ++slot) {
        const int d = dir_of(a.g, slot);
        const int L = scan_len(d, H, W), N = line_len(d, H, W), seg = L / a.g.groups;
        const T* lam = static_cast<const T*>(a.lam) + ((slot * (int64_t)B + b) * C + c) * HW;
        const T* lg = static_cast<const T*>(a.logits) + ((slot * (int64_t)B + b) * Cw + cw) * 3 * HW;
        float* hp = wsm;
        float* hc = wsm + a.lstride;
        if (lane == 0) hp[0] = hp[N + 1] = hc[0] = hc[N + 1] = 0.f;
        __syncwarp();
        const Walk wk = walk_of(d, H, W);
        for (int i = 0, gi = 0; i < L; ++i, gi = gi + 1 == seg ? 0 : gi + 1) {  // gi = i % seg
            const bool carry = gi != 0;
            for (int j = lane; j < N; j += 32) {
                const int p = wk.o + i * wk.si + j * wk.sj;
                float v = load_elt(lam, p) * load_elt(x, p);
                if (carry) {
                    const float s0 = j > 0 ? sigmoidf(load_elt(lg, p)) : 0.f;
                    const float s1 = sigmoidf(load_elt(lg, HW + p));
                    const float s2 = j < N - 1 ? sigmoidf(load_elt(lg, 2 * HW + p)) : 0.f;
                    const float num = s0 * hp[j] + s1 * hp[j + 1] + s2 * hp[j + 2];
                    v += num / (s0 + s1 + s2);
                }
                hc[j + 1] = v;
                acc[p] = slot == 0 ? v : acc[p] + v;
            }
            __syncwarp();
            float* t = hp; hp = hc; hc = t;
        }
    }
    __syncwarp();
    T* out = static_cast<T*>(a.out) + plane * HW;
    for (int q = lane; q < HW; q += 32) store_elt(out, q, acc[q]);
}

// The same forward for lines of at most 32*P positions, with the loads of line
// i+1 issued before line i is computed: lane l holds positions l + 32r (r < P)
// of the line in registers, so each line's global loads overlap the previous
// line's arithmetic instead of stalling it.
template <typename T, int P>
__global__ void __launch_bounds__(kMaxWarps * 32) generic_fwd_pipelined_kernel(FwdArgs a) {
    extern __shared__ float smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int H = a.g.H, W = a.g.W, HW = H * W, B = a.g.B, C = a.g.C;
    const int64_t plane = (int64_t)blockIdx.x * a.warps_per_cta + warp;
    if (plane >= (int64_t)B * C) return;
    float* wsm = smem + (size_t)warp * (2 * a.lstride + (a.acc_in_smem ? HW : 0));
    float* acc = a.acc_in_smem ? wsm + 2 * a.lstride : a.acc_ws + plane * HW;
    const int64_t b = plane / C, c = plane % C, cw = a.g.shared ? 0 : c;
    const int Cw = a.g.shared ? 1 : C;
    const T* x = static_cast<const T*>(a.x) + plane * HW;

    for (int slot = 0; slot < a.g.D; ++slot) {
        const int d = dir_of(a.g, slot);
        const int L = scan_len(d, H, W), N = line_len(d, H, W), seg = L / a.g.groups;
        const T* lam = static_cast<const T*>(a.lam) + ((slot * (int64_t)B + b) * C + c) * HW;
        const T* lg = static_cast<const T*>(a.logits) + ((slot * (int64_t)B + b) * Cw + cw) * 3 * HW;
        float* hp = wsm;
        float* hc = wsm + a.lstride;
        if (lane == 0) hp[0] = hp[N + 1] = hc[0] = hc[N + 1] = 0.f;
        __syncwarp();
        // inputs of the line in flight: lambda*x and the three raw tap logits
        float lx[P], g0[P], g1[P], g2[P];
        const Walk wk = walk_of(d, H, W);
        auto fetch = [&](int i, float (&flx)[P], float (&f0)[P], float (&f1)[P], float (&f2)[P]) {
#pragma unroll
            for (int r = 0; r < P; ++r) {
                const int j = lane + 32 * r;
                const int pp = j < N ? wk.o + i * wk.si + j * wk.sj : 0;  // in bounds for idle lanes
                flx[r] = load_elt(lam, pp) * load_elt(x, pp);
                f0[r] = load_elt(lg, pp);
                f1[r] = load_elt(lg, HW + pp);
                f2[r] = load_elt(lg, 2 * HW + pp);
            }
        };
        fetch(0, lx, g0, g1, g2);
        for (int i = 0, gi = 0; i < L; ++i, gi = gi + 1 == seg ? 0 : gi + 1) {  // gi = i % seg
            float nlx[P], n0[P], n1[P], n2[P];
            if (i + 1 < L) fetch(i + 1, nlx, n0, n1, n2);
            const bool carry = gi != 0;
#pragma unroll
            for (int r = 0; r < P; ++r) {
                const int j = lane + 32 * r;
                if (j < N) {
                    float v = lx[r];
                    if (carry) {
                        const float s0 = j > 0 ? sigmoidf(g0[r]) : 0.f;
                        const float s1 = sigmoidf(g1[r]);
                        const float s2 = j < N - 1 ? sigmoidf(g2[r]) : 0.f;
                        const float num = s0 * hp[j] + s1 * hp[j + 1] + s2 * hp[j + 2];
                        v += num / (s0 + s1 + s2);
                    }
                    hc[j + 1] = v;
                    const int pp = wk.o + i * wk.si + j * wk.sj;
                    acc[pp] = slot == 0 ? v : acc[pp] + v;
                }
            }
            __syncwarp();
            float* tswap = hp; hp = hc; hc = tswap;
#pragma unroll
            for (int r = 0; r < P; ++r) {
                lx[r] = nlx[r];
                g0[r] = n0[r];
                g1[r] = n1[r];
                g2[r] = n2[r];
            }
        }
    }
    __syncwarp();
    T* out = static_cast<T*>(a.out) + plane * HW;
    for (int q = lane; q < HW; q += 32) store_elt(out, q, acc[q]);
}

struct BwdArgs {
    Launch g;
    const void* x;
    const void* logits;
    const void* lam;
    const void* dout;
    void* dx;
    void* dlogits;
    void* dlam;
    float* hstore;   // [B*C][HW]: the current direction's lines, scan coordinates
    float* dx_ws;    // [B*C][HW] when the dx accumulator does not fit in smem
    unsigned long long* dlog_ws;  // [D][B][3][HW] fixed-point sums over channels (shared mode)
    int acc_in_smem;
    int warps_per_cta;
    int lstride;
};

// Backward.  With a_i = dL/dh_i in scan coordinates:
//   a_i[j] = dout_i[j] + sum_k w_{i+1}[j-k+1][k] a_{i+1}[j-k+1]   (no carry into
//            a line whose successor starts a group),
//   dx += lam a, dlam = x a, dw_k = a h_{i-1}[j+k-1],
//   dlogit_k = s_k (1 - s_k) / S (dw_k - sum_m w_m dw_m)   (valid taps; 0 else).
// The products w_k(i, j) a_i[j] of line i are kept in three shared line buffers
// so that line i-1 picks up its carry with the transposed taps.
template <typename T>
__global__ void __launch_bounds__(kMaxWarps * 32) generic_bwd_kernel(BwdArgs a) {
    extern __shared__ float smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int H = a.g.H, W = a.g.W, HW = H * W, B = a.g.B, C = a.g.C;
    const int64_t plane = (int64_t)blockIdx.x * a.warps_per_cta + warp;
    if (plane >= (int64_t)B * C) return;
    const int ls = a.lstride;
    float* wsm = smem + (size_t)warp * (6 * ls + (a.acc_in_smem ? HW : 0));
    float* dxacc = a.acc_in_smem ? wsm + 6 * ls : a.dx_ws + plane * HW;
    float* hst = a.hstore + plane * HW;
    const int64_t b = plane / C, c = plane % C, cw = a.g.shared ? 0 : c;
    const int Cw = a.g.shared ? 1 : C;
    const T* x = static_cast<const T*>(a.x) + plane * HW;
    const T* g = static_cast<const T*>(a.dout) + plane * HW;

    for (int slot = 0; slot < a.g.D; ++slot) {
        const int d = dir_of(a.g, slot);
        const int L = scan_len(d, H, W), N = line_len(d, H, W), seg = L / a.g.groups;
        const T* lam = static_cast<const T*>(a.lam) + ((slot * (int64_t)B + b) * C + c) * HW;
        const T* lg = static_cast<const T*>(a.logits) + ((slot * (int64_t)B + b) * Cw + cw) * 3 * HW;
        T* dlam = static_cast<T*>(a.dlam) + ((slot * (int64_t)B + b) * C + c) * HW;
        const Walk wk = walk_of(d, H, W);

        // 1. recompute this direction's lines into hst (scan coordinates)
        {
            float* hp = wsm;
            float* hc = wsm + ls;
            if (lane == 0) hp[0] = hp[N + 1] = hc[0] = hc[N + 1] = 0.f;
            __syncwarp();
            for (int i = 0, gi = 0; i < L; ++i, gi = gi + 1 == seg ? 0 : gi + 1) {  // gi = i % seg
                const bool carry = gi != 0;
                for (int j = lane; j < N; j += 32) {
                    const int p = wk.o + i * wk.si + j * wk.sj;
                    float v = load_elt(lam, p) * load_elt(x, p);
                    if (carry) {
                        const float s0 = j > 0 ? sigmoidf(load_elt(lg, p)) : 0.f;
                        const float s1 = sigmoidf(load_elt(lg, HW + p));
                        const float s2 = j < N - 1 ? sigmoidf(load_elt(lg, 2 * HW + p)) : 0.f;
                        v += (s0 * hp[j] + s1 * hp[j + 1] + s2 * hp[j + 2]) / (s0 + s1 + s2);
                    }
                    hc[j + 1] = v;
                    hst[i * N + j] = v;
                }
                __syncwarp();
                float* t = hp; hp = hc; hc = t;
            }
        }
        // 2. reverse scan of the adjoint
        float* qn = wsm;        // 3 buffers: products of line i+1
        float* qc = wsm + 3 * ls;  // 3 buffers: products of line i
        for (int q = lane; q < 6 * ls; q += 32) wsm[q] = 0.f;
        __syncwarp();
        // gi = i % seg, counted down from L-1 (seg divides L)
        for (int i = L - 1, gi = seg - 1; i >= 0; --i, gi = gi == 0 ? seg - 1 : gi - 1) {
            const bool carry_out = gi != 0;                      // line i reads line i-1
            const bool carry_in = (i + 1 < L) && gi != seg - 1;  // line i+1 read line i
            for (int j = lane; j < N; j += 32) {
                const int p = wk.o + i * wk.si + j * wk.sj;
                float av = load_elt(g, p);
                if (carry_in) av += qn[j + 2] + qn[ls + j + 1] + qn[2 * ls + j];
                const float lv = load_elt(lam, p), xv = load_elt(x, p);
                dxacc[p] = slot == 0 ? lv * av : dxacc[p] + lv * av;
                store_elt(dlam, p, xv * av);
                float dl0 = 0.f, dl1 = 0.f, dl2 = 0.f, q0 = 0.f, q1 = 0.f, q2 = 0.f;
                if (carry_out) {
                    const float s0 = j > 0 ? sigmoidf(load_elt(lg, p)) : 0.f;
                    const float s1 = sigmoidf(load_elt(lg, HW + p));
                    const float s2 = j < N - 1 ? sigmoidf(load_elt(lg, 2 * HW + p)) : 0.f;
                    const float r = 1.f / (s0 + s1 + s2);
                    const float w0 = s0 * r, w1 = s1 * r, w2 = s2 * r;
                    const float* hprev = hst + (i - 1) * N;
                    const float dw0 = j > 0 ? av * hprev[j - 1] : 0.f;
                    const float dw1 = av * hprev[j];
                    const float dw2 = j < N - 1 ? av * hprev[j + 1] : 0.f;
                    // dw_k - sum_m w_m dw_m = sum_m w_m (dw_k - dw_m) since the w sum to 1;
                    // the pairwise form is exactly 0 when a single tap is valid
                    const float r2 = r * r;
                    dl0 = s0 * (1.f - s0) * r2 * (s1 * (dw0 - dw1) + s2 * (dw0 - dw2));
                    dl1 = s1 * (1.f - s1) * r2 * (s0 * (dw1 - dw0) + s2 * (dw1 - dw2));
                    dl2 = s2 * (1.f - s2) * r2 * (s0 * (dw2 - dw0) + s1 * (dw2 - dw1));
                    q0 = w0 * av; q1 = w1 * av; q2 = w2 * av;
                }
                qc[j + 1] = q0;
                qc[ls + j + 1] = q1;
                qc[2 * ls + j + 1] = q2;
                if (a.g.shared) {
                    if (carry_out) {
                        unsigned long long* dw = a.dlog_ws + ((int64_t)slot * B + b) * 3 * HW;
                        if (j > 0) fix_add(dw + p, dl0);
                        fix_add(dw + HW + p, dl1);
                        if (j < N - 1) fix_add(dw + 2 * HW + p, dl2);
                    }
                } else {
                    T* dlg = static_cast<T*>(a.dlogits) + ((slot * (int64_t)B + b) * Cw + cw) * 3 * HW;
                    store_elt(dlg, p, dl0);
                    store_elt(dlg, HW + p, dl1);
                    store_elt(dlg, 2 * HW + p, dl2);
                }
            }
            __syncwarp();
            float* t = qn; qn = qc; qc = t;
        }
        __syncwarp();
    }
    T* dx = static_cast<T*>(a.dx) + plane * HW;
    for (int q = lane; q < HW; q += 32) store_elt(dx, q, dxacc[q]);
}

// The backward with the inputs of the next line in flight: lane l holds
// positions l + 32r (r < P) of a line in registers, as in the pipelined
// forward.  The recompute loads line i+1's lambda*x and tap logits before it
// computes line i; the adjoint loads line i-1's dout, lambda, x, tap logits and
// the three recomputed states it reads before it computes line i (with 8
// positions per lane the states are read where they are used, which keeps the
// kernel within its registers).  Same arithmetic in the same order as
// generic_bwd_kernel, so the same results.
template <typename T, int P>
__global__ void __launch_bounds__(kMaxWarps * 32) generic_bwd_pipelined_kernel(BwdArgs a) {
    extern __shared__ float smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int H = a.g.H, W = a.g.W, HW = H * W, B = a.g.B, C = a.g.C;
    const int64_t plane = (int64_t)blockIdx.x * a.warps_per_cta + warp;
    if (plane >= (int64_t)B * C) return;
    constexpr bool kPrefH = P <= 4;  // the states of the next line in flight too
    const int ls = a.lstride;
    float* wsm = smem + (size_t)warp * (6 * ls + (a.acc_in_smem ? HW : 0));
    float* dxacc = a.acc_in_smem ? wsm + 6 * ls : a.dx_ws + plane * HW;
    float* hst = a.hstore + plane * HW;
    const int64_t b = plane / C, c = plane % C, cw = a.g.shared ? 0 : c;
    const int Cw = a.g.shared ? 1 : C;
    const T* x = static_cast<const T*>(a.x) + plane * HW;
    const T* g = static_cast<const T*>(a.dout) + plane * HW;

    for (int slot = 0; slot < a.g.D; ++slot) {
        const int d = dir_of(a.g, slot);
        const int L = scan_len(d, H, W), N = line_len(d, H, W), seg = L / a.g.groups;
        const T* lam = static_cast<const T*>(a.lam) + ((slot * (int64_t)B + b) * C + c) * HW;
        const T* lg = static_cast<const T*>(a.logits) + ((slot * (int64_t)B + b) * Cw + cw) * 3 * HW;
        T* dlam = static_cast<T*>(a.dlam) + ((slot * (int64_t)B + b) * C + c) * HW;
        const Walk wk = walk_of(d, H, W);

        // 1. recompute this direction's lines into hst (scan coordinates)
        {
            float* hp = wsm;
            float* hc = wsm + ls;
            if (lane == 0) hp[0] = hp[N + 1] = hc[0] = hc[N + 1] = 0.f;
            __syncwarp();
            float lx[P], g0[P], g1[P], g2[P];
            auto fetch = [&](int i, float (&flx)[P], float (&f0)[P], float (&f1)[P], float (&f2)[P]) {
#pragma unroll
                for (int r = 0; r < P; ++r) {
                    const int j = lane + 32 * r;
                    const int pp = j < N ? wk.o + i * wk.si + j * wk.sj : 0;  // in bounds for idle lanes
                    flx[r] = load_elt(lam, pp) * load_elt(x, pp);
                    f0[r] = load_elt(lg, pp);
                    f1[r] = load_elt(lg, HW + pp);
                    f2[r] = load_elt(lg, 2 * HW + pp);
                }
            };
            fetch(0, lx, g0, g1, g2);
            for (int i = 0, gi = 0; i < L; ++i, gi = gi + 1 == seg ? 0 : gi + 1) {  // gi = i % seg
                float nlx[P], n0[P], n1[P], n2[P];
                if (i + 1 < L) fetch(i + 1, nlx, n0, n1, n2);
                const bool carry = gi != 0;
#pragma unroll
                for (int r = 0; r < P; ++r) {
                    const int j = lane + 32 * r;
                    if (j < N) {
                        float v = lx[r];
                        if (carry) {
                            const float s0 = j > 0 ? sigmoidf(g0[r]) : 0.f;
                            const float s1 = sigmoidf(g1[r]);
                            const float s2 = j < N - 1 ? sigmoidf(g2[r]) : 0.f;
                            v += (s0 * hp[j] + s1 * hp[j + 1] + s2 * hp[j + 2]) / (s0 + s1 + s2);
                        }
                        hc[j + 1] = v;
                        hst[i * N + j] = v;
                    }
                }
                __syncwarp();
                float* t = hp; hp = hc; hc = t;
#pragma unroll
                for (int r = 0; r < P; ++r) {
                    lx[r] = nlx[r];
                    g0[r] = n0[r];
                    g1[r] = n1[r];
                    g2[r] = n2[r];
                }
            }
        }
        // 2. reverse scan of the adjoint
        float* qn = wsm;           // 3 buffers: products of line i+1
        float* qc = wsm + 3 * ls;  // 3 buffers: products of line i
        for (int q = lane; q < 6 * ls; q += 32) wsm[q] = 0.f;
        __syncwarp();
        // line i's inputs: dout, lambda, x, the three tap logits, and the states
        // h_{i-1}[j-1], h_{i-1}[j], h_{i-1}[j+1] its tap gradients read
        float vg[P], vl[P], vx[P], t0[P], t1[P], t2[P], hm[P], hz[P], hq[P];
        auto fetch2 = [&](int i, float (&fg)[P], float (&fl)[P], float (&fx)[P], float (&f0)[P], float (&f1)[P],
                          float (&f2)[P], float (&fm)[P], float (&fz)[P], float (&fq)[P]) {
#pragma unroll
            for (int r = 0; r < P; ++r) {
                const int j = lane + 32 * r;
                const int pp = j < N ? wk.o + i * wk.si + j * wk.sj : 0;  // in bounds for idle lanes
                fg[r] = load_elt(g, pp);
                fl[r] = load_elt(lam, pp);
                fx[r] = load_elt(x, pp);
                f0[r] = load_elt(lg, pp);
                f1[r] = load_elt(lg, HW + pp);
                f2[r] = load_elt(lg, 2 * HW + pp);
                if constexpr (kPrefH) {
                    const float* hprev = hst + (i > 0 ? i - 1 : 0) * N;
                    const bool in = i > 0 && j < N;
                    fm[r] = in && j > 0 ? hprev[j - 1] : 0.f;
                    fz[r] = in ? hprev[j] : 0.f;
                    fq[r] = in && j < N - 1 ? hprev[j + 1] : 0.f;
                }
            }
        };
        fetch2(L - 1, vg, vl, vx, t0, t1, t2, hm, hz, hq);
        // gi = i % seg, counted down from L-1 (seg divides L)
        for (int i = L - 1, gi = seg - 1; i >= 0; --i, gi = gi == 0 ? seg - 1 : gi - 1) {
            float ng[P], nl[P], nx[P], n0[P], n1[P], n2[P], nm[P], nz[P], nq[P];
            if (i > 0) fetch2(i - 1, ng, nl, nx, n0, n1, n2, nm, nz, nq);
            const bool carry_out = gi != 0;                      // line i reads line i-1
            const bool carry_in = (i + 1 < L) && gi != seg - 1;  // line i+1 read line i
#pragma unroll
            for (int r = 0; r < P; ++r) {
                const int j = lane + 32 * r;
                if (j < N) {
                    const int p = wk.o + i * wk.si + j * wk.sj;
                    float av = vg[r];
                    if (carry_in) av += qn[j + 2] + qn[ls + j + 1] + qn[2 * ls + j];
                    dxacc[p] = slot == 0 ? vl[r] * av : dxacc[p] + vl[r] * av;
                    store_elt(dlam, p, vx[r] * av);
                    float dl0 = 0.f, dl1 = 0.f, dl2 = 0.f, q0 = 0.f, q1 = 0.f, q2 = 0.f;
                    if (carry_out) {
                        const float s0 = j > 0 ? sigmoidf(t0[r]) : 0.f;
                        const float s1 = sigmoidf(t1[r]);
                        const float s2 = j < N - 1 ? sigmoidf(t2[r]) : 0.f;
                        const float rr = 1.f / (s0 + s1 + s2);
                        const float w0 = s0 * rr, w1 = s1 * rr, w2 = s2 * rr;
                        float hl, hm0, hr;
                        if constexpr (kPrefH) {
                            hl = hm[r];
                            hm0 = hz[r];
                            hr = hq[r];
                        } else {
                            const float* hprev = hst + (i - 1) * N;
                            hl = j > 0 ? hprev[j - 1] : 0.f;
                            hm0 = hprev[j];
                            hr = j < N - 1 ? hprev[j + 1] : 0.f;
                        }
                        const float dw0 = j > 0 ? av * hl : 0.f;
                        const float dw1 = av * hm0;
                        const float dw2 = j < N - 1 ? av * hr : 0.f;
                        const float r2 = rr * rr;
                        dl0 = s0 * (1.f - s0) * r2 * (s1 * (dw0 - dw1) + s2 * (dw0 - dw2));
                        dl1 = s1 * (1.f - s1) * r2 * (s0 * (dw1 - dw0) + s2 * (dw1 - dw2));
                        dl2 = s2 * (1.f - s2) * r2 * (s0 * (dw2 - dw0) + s1 * (dw2 - dw1));
                        q0 = w0 * av; q1 = w1 * av; q2 = w2 * av;
                    }
                    qc[j + 1] = q0;
                    qc[ls + j + 1] = q1;
                    qc[2 * ls + j + 1] = q2;
                    if (a.g.shared) {
                        if (carry_out) {
                            unsigned long long* dw = a.dlog_ws + ((int64_t)slot * B + b) * 3 * HW;
                            if (j > 0) fix_add(dw + p, dl0);
                            fix_add(dw + HW + p, dl1);
                            if (j < N - 1) fix_add(dw + 2 * HW + p, dl2);
                        }
                    } else {
                        T* dlg = static_cast<T*>(a.dlogits) + ((slot * (int64_t)B + b) * Cw + cw) * 3 * HW;
                        store_elt(dlg, p, dl0);
                        store_elt(dlg, HW + p, dl1);
                        store_elt(dlg, 2 * HW + p, dl2);
                    }
                }
            }
            __syncwarp();
            float* t = qn; qn = qc; qc = t;
#pragma unroll
            for (int r = 0; r < P; ++r) {
                vg[r] = ng[r]; vl[r] = nl[r]; vx[r] = nx[r];
                t0[r] = n0[r]; t1[r] = n1[r]; t2[r] = n2[r];
                if constexpr (kPrefH) {
                    hm[r] = nm[r]; hz[r] = nz[r]; hq[r] = nq[r];
                }
            }
        }
        __syncwarp();
    }
    T* dx = static_cast<T*>(a.dx) + plane * HW;
    for (int q = lane; q < HW; q += 32) store_elt(dx, q, dxacc[q]);
}

__global__ void zero_fix_kernel(unsigned long long* p, int64_t n) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
        p[i] = 0ull;
}

template <typename T>
__global__ void convert_fix_kernel(const unsigned long long* src, T* dst, int64_t n) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
        store_elt(dst, i, fix_value(src[i]));
}

struct Plan {
    int wpc;          // warps per CTA
    int acc_in_smem;
    int lstride;
    size_t smem;      // dynamic smem bytes per CTA
};

Plan plan_for(const Problem& p, const DeviceInfo& dev, int line_bufs) {
    Plan pl;
    const int nmax = p.g.H > p.g.W ? p.g.H : p.g.W;
    pl.lstride = nmax + 2;
    const size_t lines = (size_t)line_bufs * pl.lstride * sizeof(float);
    const size_t acc = (size_t)p.HW * sizeof(float);
    const size_t budget = dev.max_smem_optin < kSmemBudget ? (size_t)dev.max_smem_optin : (size_t)kSmemBudget;
    if (lines + acc <= budget) {
        pl.acc_in_smem = 1;
        pl.wpc = (int)(budget / (lines + acc));
    } else {
        pl.acc_in_smem = 0;
        pl.wpc = (int)(budget / lines);
    }
    if (pl.wpc > kMaxWarps) pl.wpc = kMaxWarps;
    // spread the planes over the SMs before stacking them in a CTA: with fewer
    // planes than 8 per SM, CTAs of fewer warps (one warp is one plane)
    const int64_t per_sm = (p.planes + dev.sm_count - 1) / (dev.sm_count > 0 ? dev.sm_count : 1);
    if ((int64_t)pl.wpc > per_sm) pl.wpc = (int)per_sm;
    if (pl.wpc < 1) pl.wpc = 1;
    if ((int64_t)pl.wpc > p.planes) pl.wpc = (int)p.planes;
    pl.smem = (size_t)pl.wpc * (lines + (pl.acc_in_smem ? acc : 0));
    return pl;
}

bool lines_fit(const Problem& p, const DeviceInfo& dev, int line_bufs) {
    const int nmax = p.g.H > p.g.W ? p.g.H : p.g.W;
    return (size_t)line_bufs * (nmax + 2) * sizeof(float) <= (size_t)dev.max_smem_optin;
}

gspn_status cuda_status(cudaError_t e) { return e == cudaSuccess ? GSPN_OK : GSPN_ERR_CUDA; }

int64_t grid_for(int64_t n, int threads) {
    int64_t g = (n + threads - 1) / threads;
    if (g > 65535) g = 65535;
    if (g < 1) g = 1;
    return g;
}

}  // namespace

size_t generic_fwd_workspace(const Problem& p, const DeviceInfo& dev) {
    Plan pl = plan_for(p, dev, 2);
    return pl.acc_in_smem ? 0 : align_up((size_t)p.planes * p.HW * sizeof(float), kWsAlign);
}

gspn_status generic_fwd(const Problem& p, const DeviceInfo& dev, const void* x, const void* logits,
                        const void* lam, void* out, void* ws, cudaStream_t s) {
    if (!lines_fit(p, dev, 2)) return GSPN_ERR_UNSUPPORTED;
    Plan pl = plan_for(p, dev, 2);
    FwdArgs a;
    a.g = p.g; a.x = x; a.logits = logits; a.lam = lam; a.out = out;
    a.acc_ws = static_cast<float*>(ws);
    a.acc_in_smem = pl.acc_in_smem; a.warps_per_cta = pl.wpc; a.lstride = pl.lstride;
    const int64_t grid = (p.planes + pl.wpc - 1) / pl.wpc;
    if (grid > 0x7fffffff) return GSPN_ERR_UNSUPPORTED;
    const int nmax = p.g.H > p.g.W ? p.g.H : p.g.W;
    const bool f32 = p.d.dtype == GSPN_F32;
    // lines of up to 256 positions: the pipelined kernel with 1, 2, 4 or 8 positions per lane
    const void* fn;
    int slot;
    if (nmax <= 32) {
        fn = f32 ? (const void*)generic_fwd_pipelined_kernel<float, 1>
                 : (const void*)generic_fwd_pipelined_kernel<__nv_bfloat16, 1>;
        slot = f32 ? 11 : 12;
    } else if (nmax <= 64) {
        fn = f32 ? (const void*)generic_fwd_pipelined_kernel<float, 2>
                 : (const void*)generic_fwd_pipelined_kernel<__nv_bfloat16, 2>;
        slot = f32 ? 13 : 14;
    } else if (nmax <= 128) {
        fn = f32 ? (const void*)generic_fwd_pipelined_kernel<float, 4>
                 : (const void*)generic_fwd_pipelined_kernel<__nv_bfloat16, 4>;
        slot = f32 ? 15 : 16;
    } else if (nmax <= 256) {
        fn = f32 ? (const void*)generic_fwd_pipelined_kernel<float, 8>
                 : (const void*)generic_fwd_pipelined_kernel<__nv_bfloat16, 8>;
        slot = f32 ? 39 : 40;
    } else {
        fn = f32 ? (const void*)generic_fwd_kernel<float> : (const void*)generic_fwd_kernel<__nv_bfloat16>;
        slot = f32 ? 0 : 1;
    }
    cudaError_t e = ensure_smem_attr(fn, (int)pl.smem, slot);
    if (e != cudaSuccess) return GSPN_ERR_CUDA;
    void* args[] = {&a};
    e = cudaLaunchKernel(fn, dim3((unsigned)grid), dim3(pl.wpc * 32), args, pl.smem, s);
    return cuda_status(e);
}

namespace {
struct BwdWs {
    size_t hstore, dx_ws, dlog_ws, total;
};
BwdWs bwd_ws_layout(const Problem& p, const DeviceInfo& dev) {
    Plan pl = plan_for(p, dev, 6);
    BwdWs w;
    const size_t plane_f = (size_t)p.planes * p.HW * sizeof(float);
    w.hstore = 0;
    size_t off = align_up(plane_f, kWsAlign);
    w.dx_ws = off;
    if (!pl.acc_in_smem) off += align_up(plane_f, kWsAlign);
    w.dlog_ws = off;
    if (p.g.shared) off += align_up((size_t)p.g.D * p.g.B * 3 * p.HW * sizeof(unsigned long long), kWsAlign);
    w.total = off;
    return w;
}
}  // namespace

size_t generic_bwd_workspace(const Problem& p, const DeviceInfo& dev) { return bwd_ws_layout(p, dev).total; }

int generic_bwd_launches(const Problem& p) { return p.g.shared ? 3 : 1; }

gspn_status generic_bwd(const Problem& p, const DeviceInfo& dev, const void* x, const void* logits,
                        const void* lam, const void* dout, void* dx, void* dlogits, void* dlam, void* ws,
                        cudaStream_t s) {
    if (!lines_fit(p, dev, 6)) return GSPN_ERR_UNSUPPORTED;
    Plan pl = plan_for(p, dev, 6);
    BwdWs lay = bwd_ws_layout(p, dev);
    char* w = static_cast<char*>(ws);
    BwdArgs a;
    a.g = p.g; a.x = x; a.logits = logits; a.lam = lam; a.dout = dout;
    a.dx = dx; a.dlogits = dlogits; a.dlam = dlam;
    a.hstore = reinterpret_cast<float*>(w + lay.hstore);
    a.dx_ws = reinterpret_cast<float*>(w + lay.dx_ws);
    a.dlog_ws = reinterpret_cast<unsigned long long*>(w + lay.dlog_ws);
    a.acc_in_smem = pl.acc_in_smem; a.warps_per_cta = pl.wpc; a.lstride = pl.lstride;
    const int64_t nlog = (int64_t)p.g.D * p.g.B * 3 * p.HW;
    if (p.g.shared) {
        zero_fix_kernel<<<(unsigned)grid_for(nlog, 256), 256, 0, s>>>(a.dlog_ws, nlog);
        cudaError_t e0 = cudaGetLastError();
        if (e0 != cudaSuccess) return GSPN_ERR_CUDA;
    }
    const int64_t grid = (p.planes + pl.wpc - 1) / pl.wpc;
    if (grid > 0x7fffffff) return GSPN_ERR_UNSUPPORTED;
    // lines of up to 256 positions: the pipelined kernel with 1, 2, 4 or 8 positions per lane
    const int nmax = p.g.H > p.g.W ? p.g.H : p.g.W;
    const bool f32 = p.d.dtype == GSPN_F32;
    const void* fn;
    int slot;
    if (nmax <= 32) {
        fn = f32 ? (const void*)generic_bwd_pipelined_kernel<float, 1>
                 : (const void*)generic_bwd_pipelined_kernel<__nv_bfloat16, 1>;
        slot = f32 ? 4 : 5;
    } else if (nmax <= 64) {
        fn = f32 ? (const void*)generic_bwd_pipelined_kernel<float, 2>
                 : (const void*)generic_bwd_pipelined_kernel<__nv_bfloat16, 2>;
        slot = f32 ? 6 : 7;
    } else if (nmax <= 128) {
        fn = f32 ? (const void*)generic_bwd_pipelined_kernel<float, 4>
                 : (const void*)generic_bwd_pipelined_kernel<__nv_bfloat16, 4>;
        slot = f32 ? 30 : 31;
    } else if (nmax <= 256) {
        fn = f32 ? (const void*)generic_bwd_pipelined_kernel<float, 8>
                 : (const void*)generic_bwd_pipelined_kernel<__nv_bfloat16, 8>;
        slot = f32 ? 41 : 42;
    } else {
        fn = f32 ? (const void*)generic_bwd_kernel<float> : (const void*)generic_bwd_kernel<__nv_bfloat16>;
        slot = f32 ? 2 : 3;
    }
    cudaError_t e = ensure_smem_attr(fn, (int)pl.smem, slot);
    if (e != cudaSuccess) return GSPN_ERR_CUDA;
    void* kargs[] = {&a};
    e = cudaLaunchKernel(fn, dim3((unsigned)grid), dim3(pl.wpc * 32), kargs, pl.smem, s);
    if (e != cudaSuccess) return GSPN_ERR_CUDA;
    e = cudaGetLastError();
    if (e != cudaSuccess) return GSPN_ERR_CUDA;
    if (p.g.shared) {
        if (p.d.dtype == GSPN_F32)
            convert_fix_kernel<float><<<(unsigned)grid_for(nlog, 256), 256, 0, s>>>(
                a.dlog_ws, static_cast<float*>(dlogits), nlog);
        else
            convert_fix_kernel<__nv_bfloat16><<<(unsigned)grid_for(nlog, 256), 256, 0, s>>>(
                a.dlog_ws, static_cast<__nv_bfloat16*>(dlogits), nlog);
        e = cudaGetLastError();
        if (e != cudaSuccess) return GSPN_ERR_CUDA;
    }
    return GSPN_OK;
}

}  // namespace gspn
