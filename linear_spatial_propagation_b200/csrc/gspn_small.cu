// gspn_small.cu -- GSPN forward and backward for planes of at most 64x64, in
// any dtype, direction set, local-group count and weight mode (per-channel
// taps in particular: the tiny-backbone 56x56 and local 28x28 stages of
// "Parallel Sequence Modeling via Generalized Spatial Propagation Network").
//
// One CTA per (b, c) plane, one warp per enabled direction: the four scans of
// a plane (Key design 2) run side by side instead of one after the other, and
// each keeps its own fp32 copy of the plane in shared memory, summed in
// direction order at the end (the merge), so the result does not depend on
// timing.  Lane l holds positions l (and l+32: P = 2) of a line; the previous line sits
// in a shared line buffer with a zero halo, so tap k of position j reads slot
// j+k.  The tap weights are recomputed from the logits where they are used:
// s_k = sigmoid(logit_k) on the taps whose source lies in the line, w_k =
// s_k / sum s (Key design 1).
//
// Inputs are read 4 lines at a time (8 for fp32 with two positions per lane): each lane
// loads its positions' values of those lines in one go.  For a row scan the lanes of a warp read along a
// row; for a column scan each lane reads the neighbouring pixels of its row,
// with 8-byte loads where the pieces are aligned.
//
// Backward: per direction, the lines are recomputed into shared memory, then
// the adjoint runs from the last line to the first with the transposed taps
// ("GSPN-2: Efficient Parallel Sequence Modeling", Backward Benchmark):
//   a_i[j] = G_i[j] + sum_k w_{i+1}[j-k+1][k] a_{i+1}[j-k+1]  (no carry into a
//            line whose successor starts a group),
//   dx += lambda a, dlambda = x a, dw_k = a h_{i-1}[j+k-1],
//   dlogit_k = s_k (1 - s_k) / S (dw_k - sum_m w_m dw_m)  (valid taps; 0 else).
// dx is summed over the directions in shared memory, in direction order.
#include "gspn_internal.h"

namespace gspn {

namespace {

constexpr int kLS = 66;    // line buffer: up to 64 positions + a zero halo at each end
// lines whose inputs are loaded together: 8 for fp32 with two positions per
// lane, 4 otherwise.  With one position per lane that means fewer registers and
// more CTAs per SM for the many small planes; for bf16 with two positions it
// was measured faster in the forward (64x64: 145 -> 119 us) and keeps the
// backward's six input planes within the 168 registers of 3 CTAs per SM.  fp32
// with two positions is faster with 8 (56x56 forward: 93 against 159 us).
template <int P, int BYTES>
__host__ __device__ constexpr int chunk_of() { return P == 2 && BYTES == 4 ? 8 : 4; }
constexpr int kSmallSmemCap = 200 * 1024;

struct SmallArgs {
    Launch g;
    const void* x;
    const void* logits;
    const void* lam;
    const void* dout;
    void* out;      // forward
    void* dx;       // backward
    void* dlogits;
    void* dlam;
    unsigned long long* dlog_ws;  // backward, shared taps: fixed-point sums over channels [D][B][3][HW]
};

// The sigmoids of the valid taps of position j from the raw logits.  These
// kernels compute the taps at every use, so the divisions take the fast
// reciprocal path of __fdividef (a couple of ulp) instead of IEEE division;
// its result is 0 once 1 + e^-z passes 2^126 (logits below about -87), where
// the sigmoid is below 1e-38 anyway.
__device__ __forceinline__ float fast_sigmoid(float z) { return __fdividef(1.f, 1.f + __expf(-z)); }
__device__ __forceinline__ void taps(float g0, float g1, float g2, int j, int N, float& s0, float& s1, float& s2) {
    s0 = j > 0 ? fast_sigmoid(g0) : 0.f;
    s1 = fast_sigmoid(g1);
    s2 = j < N - 1 ? fast_sigmoid(g2) : 0.f;
}

// For a column scan the CH values of one position over lines i0, i0+1, ...
// (DOWN: i0, i0-1, ...) are CH neighbouring pixels of one row.  This reads
// them with 8-byte loads and returns true when the piece is whole and aligned.
template <int CH, bool DOWN, typename T>
__device__ __forceinline__ bool load_row_piece(const T* src, int d, int W, int L, int i0, int j, float (&v)[CH]) {
    constexpr int kPer = 8 / (int)sizeof(T);  // elements per 8-byte load
    static_assert(CH % kPer == 0, "whole 8-byte loads");
    const int ilo = DOWN ? i0 - (CH - 1) : i0;  // the lowest line of the chunk
    if (ilo < 0 || ilo + CH > L) return false;
    // pixels of lines ilo..ilo+7: ascending columns for left->right, descending for right->left
    const int first = d == L2R ? j * W + ilo : j * W + (W - CH - ilo);
    if ((reinterpret_cast<uintptr_t>(src + first) & 7u) != 0) return false;
    float t[CH];
#pragma unroll
    for (int u = 0; u < CH / kPer; ++u) {
        const uint2 w = __ldg(reinterpret_cast<const uint2*>(src + first) + u);
        if constexpr (sizeof(T) == 4) {
            t[2 * u] = __uint_as_float(w.x);
            t[2 * u + 1] = __uint_as_float(w.y);
        } else {
            t[4 * u] = __uint_as_float(w.x << 16);
            t[4 * u + 1] = __uint_as_float(w.x & 0xffff0000u);
            t[4 * u + 2] = __uint_as_float(w.y << 16);
            t[4 * u + 3] = __uint_as_float(w.y & 0xffff0000u);
        }
    }
    // t[m] is line ilo + m (left->right) or ilo + CH-1 - m (right->left); two
    // branches keep every index a compile-time constant
    if (d == L2R) {
#pragma unroll
        for (int e = 0; e < CH; ++e) v[e] = t[DOWN ? CH - 1 - e : e];
    } else {
#pragma unroll
        for (int e = 0; e < CH; ++e) v[e] = t[DOWN ? e : CH - 1 - e];
    }
    return true;
}

// The reverse of load_row_piece for the bf16 backward's outputs of a column
// scan.  Line itop - e (e < CH, lines below 0 absent) of position j in
// direction d (left->right or right->left) is bf16 value e of v, two per word
// (even e in the low half), so a tensor's CH values of one chunk are CH
// neighbouring pixels of row j.  They leave as one 8-byte store per 4 when
// the piece is whole and aligned, else one element at a time.
template <int CH>
__device__ __forceinline__ void put_bf16(uint32_t (&v)[CH / 2], int e, float x) {
    const uint32_t b = __bfloat16_as_ushort(__float2bfloat16_rn(x));
    v[e >> 1] = (e & 1) ? (v[e >> 1] | (b << 16)) : b;
}
template <int CH>
__device__ __forceinline__ void store_row_piece(__nv_bfloat16* dst, int d, int W, int itop, int j,
                                                const uint32_t (&v)[CH / 2]) {
    static_assert(CH % 4 == 0, "whole 8-byte stores");
    const int ilo = itop - (CH - 1);
    // address order: left->right holds line ilo + m at element m (e = CH-1-m),
    // right->left line itop - m (e = m)
    const int first = d == L2R ? j * W + ilo : j * W + (W - 1 - itop);
    if (ilo >= 0 && (reinterpret_cast<uintptr_t>(dst + first) & 7u) == 0) {
        uint32_t w[CH / 2];
        if (d == L2R) {
#pragma unroll
            for (int u = 0; u < CH / 2; ++u) w[u] = __byte_perm(v[CH / 2 - 1 - u], 0, 0x1032);  // halves swapped
        } else {
#pragma unroll
            for (int u = 0; u < CH / 2; ++u) w[u] = v[u];
        }
#pragma unroll
        for (int u = 0; u < CH / 4; ++u) reinterpret_cast<uint2*>(dst + first)[u] = make_uint2(w[2 * u], w[2 * u + 1]);
    } else {
        unsigned short* const o = reinterpret_cast<unsigned short*>(dst);
#pragma unroll
        for (int e = 0; e < CH; ++e) {
            const int i = itop - e;
            if (i >= 0) o[d == L2R ? j * W + i : j * W + (W - 1 - i)] = (unsigned short)(v[e >> 1] >> (16 * (e & 1)));
        }
    }
}

// The chunk's inputs of lane positions j = lane + 32r: NT planes (x, lambda, the
// three logits, and dout in the backward) at lines i0 +- e.  Column scans use the
// row-piece loads when every plane's piece is aligned (the planes share the
// row offsets, so one test decides); otherwise one pixel index per (r, e) serves
// all planes.
template <int CH, bool DOWN, int P, int NT, typename T>
__device__ __forceinline__ void load_chunk(const T* const (&src)[NT], int d, const Walk& wk, int W, int L, int N,
                                           int i0, int lane, float (&v)[NT][P][CH]) {
#pragma unroll
    for (int r = 0; r < P; ++r) {
        const int j = lane + 32 * r;
        bool done = false;
        if ((d == L2R || d == R2L) && j < N) {
            done = true;
#pragma unroll
            for (int k = 0; k < NT; ++k) done = done && load_row_piece<CH, DOWN>(src[k], d, W, L, i0, j, v[k][r]);
        }
        if (!done) {
#pragma unroll
            for (int e = 0; e < CH; ++e) {
                const int i = DOWN ? i0 - e : i0 + e;
                const bool in = j < N && i >= 0 && i < L;
                const int p = in ? wk.o + i * wk.si + j * wk.sj : 0;  // in bounds for idle lanes
#pragma unroll
                for (int k = 0; k < NT; ++k) v[k][r][e] = in ? load_elt(src[k], p) : 0.f;
            }
        }
    }
}

template <typename T, int P>
__global__ void __launch_bounds__(128) small_fwd_kernel(SmallArgs a) {
    constexpr int CH = chunk_of<P, (int)sizeof(T)>();
    extern __shared__ float smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int H = a.g.H, W = a.g.W, HW = H * W, B = a.g.B, C = a.g.C, D = a.g.D;
    const int64_t plane = blockIdx.x;
    const int64_t b = plane / C, c = plane % C, cw = a.g.shared ? 0 : c;
    const int Cw = a.g.shared ? 1 : C;
    float* const acc = smem + (size_t)warp * HW;  // this direction's copy of the plane
    float* hp = smem + (size_t)D * HW + (size_t)warp * 2 * kLS;
    float* hc = hp + kLS;

    const int slot = warp, d = dir_of(a.g, slot);
    const int L = scan_len(d, H, W), N = line_len(d, H, W), seg = L / a.g.groups;
    const T* x = static_cast<const T*>(a.x) + plane * HW;
    const T* lam = static_cast<const T*>(a.lam) + ((slot * (int64_t)B + b) * C + c) * HW;
    const T* lg = static_cast<const T*>(a.logits) + ((slot * (int64_t)B + b) * Cw + cw) * 3 * HW;
    const T* const srcs[5] = {x, lam, lg, lg + HW, lg + 2 * HW};
    if (lane == 0) hp[0] = hp[N + 1] = hc[0] = hc[N + 1] = 0.f;
    __syncwarp();
    const Walk wk = walk_of(d, H, W);
    int pj[P];  // plane offset of this lane's positions on line 0
#pragma unroll
    for (int r = 0; r < P; ++r) pj[r] = wk.o + (lane + 32 * r) * wk.sj;

    int gi = 0;  // the line's index within its local group (i % seg, kept by counting)
    for (int i0 = 0; i0 < L; i0 += CH) {
        float vin[5][P][CH];
        load_chunk<CH, false, P, 5>(srcs, d, wk, W, L, N, i0, lane, vin);
        auto& vx = vin[0];
        auto& vl = vin[1];
        auto& v0 = vin[2];
        auto& v1 = vin[3];
        auto& v2 = vin[4];
#pragma unroll
        for (int e = 0; e < CH; ++e) {
            const int i = i0 + e;
            if (i >= L) break;
            const bool carry = gi != 0;
            gi = gi + 1 == seg ? 0 : gi + 1;
            const int pi = i * wk.si;
#pragma unroll
            for (int r = 0; r < P; ++r) {
                const int j = lane + 32 * r;
                if (j < N) {
                    float v = vl[r][e] * vx[r][e];
                    if (carry) {
                        float s0, s1, s2;
                        taps(v0[r][e], v1[r][e], v2[r][e], j, N, s0, s1, s2);
                        v += __fdividef(s0 * hp[j] + s1 * hp[j + 1] + s2 * hp[j + 2], s0 + s1 + s2);
                    }
                    hc[j + 1] = v;
                    acc[pj[r] + pi] = v;
                }
            }
            __syncwarp();
            float* t = hp;
            hp = hc;
            hc = t;
        }
    }
    __syncthreads();
    // the merge: the directions' planes summed in direction order, one store per pixel
    T* out = static_cast<T*>(a.out) + plane * HW;
    for (int q = threadIdx.x; q < HW; q += blockDim.x) {
        float s = smem[q];
        for (int k = 1; k < D; ++k) s += smem[(size_t)k * HW + q];
        store_elt(out, q, s);
    }
}

// (with one position per lane, at most 80 registers for fp32: 6 CTAs per SM;
// bf16 holds the row pieces as well and takes 5)
template <typename T, int P>
__global__ void __launch_bounds__(128, P == 2 ? 3 : sizeof(T) == 2 ? 5 : 6) small_bwd_kernel(SmallArgs a) {
    constexpr int CH = chunk_of<P, (int)sizeof(T)>();
    extern __shared__ float smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int H = a.g.H, W = a.g.W, HW = H * W, B = a.g.B, C = a.g.C, D = a.g.D;
    const int64_t plane = blockIdx.x;
    const int64_t b = plane / C, c = plane % C, cw = a.g.shared ? 0 : c;
    const int Cw = a.g.shared ? 1 : C;
    // this direction's lines in scan coordinates (line i at i * N).  With two
    // positions per lane (lines of 33..64) its share of dx then takes the place
    // of the lines the adjoint has left (line i's h is last read as the
    // predecessor of line i+1), so a plane needs half the shared memory and
    // more CTAs fit; with one per lane (where registers, not shared memory,
    // bound the CTAs per SM) dx has planes of its own, in image coordinates.
    constexpr bool kDxInPlace = P == 2;
    float* const hst = smem + (size_t)warp * HW;
    float* const dxacc = smem + (size_t)(D + warp) * HW;  // one position per lane only
    float* const lb = smem + (size_t)(kDxInPlace ? 1 : 2) * D * HW + (size_t)warp * 6 * kLS;  // line buffers

    const int slot = warp, d = dir_of(a.g, slot);
    const int L = scan_len(d, H, W), N = line_len(d, H, W), seg = L / a.g.groups;
    const T* x = static_cast<const T*>(a.x) + plane * HW;
    const T* g = static_cast<const T*>(a.dout) + plane * HW;
    const T* lam = static_cast<const T*>(a.lam) + ((slot * (int64_t)B + b) * C + c) * HW;
    const T* lg = static_cast<const T*>(a.logits) + ((slot * (int64_t)B + b) * Cw + cw) * 3 * HW;
    T* dlam = static_cast<T*>(a.dlam) + ((slot * (int64_t)B + b) * C + c) * HW;
    T* dlg = static_cast<T*>(a.dlogits) + ((slot * (int64_t)B + b) * Cw + cw) * 3 * HW;
    const T* const srcs[5] = {x, lam, lg, lg + HW, lg + 2 * HW};
    const T* const srcs6[6] = {g, x, lam, lg, lg + HW, lg + 2 * HW};
    // A column scan's dlambda and dlogits of one position and chunk are
    // neighbouring pixels of a row.  In bf16 they are gathered and written as
    // 8-byte pieces (4 lines), instead of one scattered 2-byte element per
    // lane and line; fp32 keeps the element stores (measured faster there).
    constexpr bool kPieces = sizeof(T) == 2;
    const bool col = d == L2R || d == R2L;

    const Walk wk = walk_of(d, H, W);

    // 1. recompute this direction's lines into shared memory
    {
        float* hp = lb;
        float* hc = lb + kLS;
        if (lane == 0) hp[0] = hp[N + 1] = hc[0] = hc[N + 1] = 0.f;
        __syncwarp();
        int gi = 0;  // i % seg, kept by counting
        for (int i0 = 0; i0 < L; i0 += CH) {
            float vin[5][P][CH];
            load_chunk<CH, false, P, 5>(srcs, d, wk, W, L, N, i0, lane, vin);
            auto& vx = vin[0];
            auto& vl = vin[1];
            auto& v0 = vin[2];
            auto& v1 = vin[3];
            auto& v2 = vin[4];
#pragma unroll
            for (int e = 0; e < CH; ++e) {
                const int i = i0 + e;
                if (i >= L) break;
                const bool carry = gi != 0;
                gi = gi + 1 == seg ? 0 : gi + 1;
#pragma unroll
                for (int r = 0; r < P; ++r) {
                    const int j = lane + 32 * r;
                    if (j < N) {
                        float v = vl[r][e] * vx[r][e];
                        if (carry) {
                            float s0, s1, s2;
                            taps(v0[r][e], v1[r][e], v2[r][e], j, N, s0, s1, s2);
                            v += __fdividef(s0 * hp[j] + s1 * hp[j + 1] + s2 * hp[j + 2], s0 + s1 + s2);
                        }
                        hc[j + 1] = v;
                        hst[i * N + j] = v;
                    }
                }
                __syncwarp();
                float* t = hp;
                hp = hc;
                hc = t;
            }
        }
    }

    // 2. the adjoint from the last line to the first; the products w_k a of the
    //    line below wait in three line buffers (zero halos) for its predecessor
    float* qn = lb;
    float* qc = lb + 3 * kLS;
    for (int q = lane; q < 6 * kLS; q += 32) lb[q] = 0.f;
    __syncwarp();
    int gi = seg - 1;  // i % seg for i = L-1 (seg divides L), kept by counting down
    for (int it = 0; it < L; it += CH) {
        // lines i = L-1-it-e, e < CH
        float vin[6][P][CH];
        load_chunk<CH, true, P, 6>(srcs6, d, wk, W, L, N, L - 1 - it, lane, vin);
        auto& vg = vin[0];
        auto& vx = vin[1];
        auto& vl = vin[2];
        auto& v0 = vin[3];
        auto& v1 = vin[4];
        auto& v2 = vin[5];
        // column scans in bf16: the chunk's dlambda and dlogits, written as row pieces at its end
        uint32_t cl[P][CH / 2], cg0[P][CH / 2], cg1[P][CH / 2], cg2[P][CH / 2];
#pragma unroll
        for (int e = 0; e < CH; ++e) {
            const int i = L - 1 - it - e;
            if (i < 0) break;
            const bool carry_out = gi != 0;                   // line i reads line i-1
            const bool carry_in = (i + 1 < L) && gi != seg - 1;  // line i+1 read line i
            gi = gi == 0 ? seg - 1 : gi - 1;
            const int pi = wk.o + i * wk.si;
#pragma unroll
            for (int r = 0; r < P; ++r) {
                const int j = lane + 32 * r;
                if (j < N) {
                    const int p = pi + j * wk.sj;
                    float av = vg[r][e];
                    if (carry_in) av += qn[j + 2] + qn[kLS + j + 1] + qn[2 * kLS + j];
                    const float dxv = vl[r][e] * av;
                    if (kPieces && col)
                        put_bf16<CH>(cl[r], e, vx[r][e] * av);
                    else
                        store_elt(dlam, p, vx[r][e] * av);
                    float dl0 = 0.f, dl1 = 0.f, dl2 = 0.f, q0 = 0.f, q1 = 0.f, q2 = 0.f;
                    if (carry_out) {
                        float s0, s1, s2;
                        taps(v0[r][e], v1[r][e], v2[r][e], j, N, s0, s1, s2);
                        const float rs = __fdividef(1.f, s0 + s1 + s2);
                        const float* hprev = hst + (i - 1) * N;
                        const float dw0 = j > 0 ? av * hprev[j - 1] : 0.f;
                        const float dw1 = av * hprev[j];
                        const float dw2 = j < N - 1 ? av * hprev[j + 1] : 0.f;
                        // dw_k - sum_m w_m dw_m = sum_m w_m (dw_k - dw_m), since the w sum to 1
                        const float r2 = rs * rs;
                        dl0 = s0 * (1.f - s0) * r2 * (s1 * (dw0 - dw1) + s2 * (dw0 - dw2));
                        dl1 = s1 * (1.f - s1) * r2 * (s0 * (dw1 - dw0) + s2 * (dw1 - dw2));
                        dl2 = s2 * (1.f - s2) * r2 * (s0 * (dw2 - dw0) + s1 * (dw2 - dw1));
                        q0 = s0 * rs * av;
                        q1 = s1 * rs * av;
                        q2 = s2 * rs * av;
                    }
                    qc[j + 1] = q0;
                    qc[kLS + j + 1] = q1;
                    qc[2 * kLS + j + 1] = q2;
                    if constexpr (kDxInPlace)
                        hst[i * N + j] = dxv;  // h of line i is dead: line i+1 has been processed
                    else
                        dxacc[p] = dxv;
                    if (a.g.shared) {
                        if (carry_out) {
                            unsigned long long* dw = a.dlog_ws + ((int64_t)slot * B + b) * 3 * HW;
                            if (j > 0) fix_add(dw + p, dl0);
                            fix_add(dw + HW + p, dl1);
                            if (j < N - 1) fix_add(dw + 2 * HW + p, dl2);
                        }
                    } else if (kPieces && col) {
                        put_bf16<CH>(cg0[r], e, dl0);
                        put_bf16<CH>(cg1[r], e, dl1);
                        put_bf16<CH>(cg2[r], e, dl2);
                    } else {
                        store_elt(dlg, p, dl0);
                        store_elt(dlg, HW + p, dl1);
                        store_elt(dlg, 2 * HW + p, dl2);
                    }
                }
            }
            __syncwarp();
            float* t = qn;
            qn = qc;
            qc = t;
        }
        if constexpr (kPieces) {
            if (col) {
                __nv_bfloat16* const bl = reinterpret_cast<__nv_bfloat16*>(dlam);
                __nv_bfloat16* const bg = reinterpret_cast<__nv_bfloat16*>(dlg);
#pragma unroll
                for (int r = 0; r < P; ++r) {
                    const int j = lane + 32 * r;
                    if (j < N) {
                        store_row_piece<CH>(bl, d, W, L - 1 - it, j, cl[r]);
                        if (!a.g.shared) {
                            store_row_piece<CH>(bg, d, W, L - 1 - it, j, cg0[r]);
                            store_row_piece<CH>(bg + HW, d, W, L - 1 - it, j, cg1[r]);
                            store_row_piece<CH>(bg + 2 * HW, d, W, L - 1 - it, j, cg2[r]);
                        }
                    }
                }
            }
        }
    }
    __syncthreads();
    // dx: the directions' shares summed in direction order
    T* dx = static_cast<T*>(a.dx) + plane * HW;
    if constexpr (kDxInPlace) {
        // share k sits in scan coordinates of its direction: pixel (row, col) at
        // line i, position j
        for (int q = threadIdx.x; q < HW; q += blockDim.x) {
            const int row = q / W, col = q - row * W;
            float s = 0.f;
            for (int k = 0; k < D; ++k) {
                const int dk = dir_of(a.g, k);
                const int idx = dk == T2B   ? row * W + col
                                : dk == B2T ? (H - 1 - row) * W + col
                                : dk == L2R ? col * H + row
                                            : (W - 1 - col) * H + row;
                s = k == 0 ? smem[(size_t)k * HW + idx] : s + smem[(size_t)k * HW + idx];
            }
            store_elt(dx, q, s);
        }
    } else {
        for (int q = threadIdx.x; q < HW; q += blockDim.x) {
            float s = smem[(size_t)D * HW + q];
            for (int k = 1; k < D; ++k) s += smem[(size_t)(D + k) * HW + q];
            store_elt(dx, q, s);
        }
    }
}

__global__ void small_zero_kernel(unsigned long long* p, int64_t n) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
        p[i] = 0ull;
}

template <typename T>
__global__ void small_convert_kernel(const unsigned long long* src, T* dst, int64_t n) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
        store_elt(dst, i, fix_value(src[i]));
}

size_t fwd_smem(const Problem& p) { return ((size_t)p.g.D * p.HW + (size_t)p.g.D * 2 * kLS) * sizeof(float); }
// one plane per direction with two positions per lane (dx in place of the dead
// lines), two with one per lane (lines of at most 32 positions)
size_t bwd_smem(const Problem& p) {
    const bool one = (p.g.H > p.g.W ? p.g.H : p.g.W) <= 32;
    return ((size_t)(one ? 2 : 1) * p.g.D * p.HW + (size_t)p.g.D * 6 * kLS) * sizeof(float);
}
unsigned grid_1d(int64_t n) {
    const int64_t g = (n + 255) / 256;
    return (unsigned)(g < 4096 ? (g > 0 ? g : 1) : 4096);
}

}  // namespace

// (the shared-memory cap is below what every sm_100 device lets a block opt in to)
bool small_eligible(const Problem& p, int backward) {
    if (p.g.H > 64 || p.g.W > 64 || p.planes > 0x7fffffff) return false;
    return (backward ? bwd_smem(p) : fwd_smem(p)) <= (size_t)kSmallSmemCap;
}

size_t small_bwd_workspace(const Problem& p) {
    return p.g.shared ? align_up((size_t)p.g.D * p.g.B * 3 * p.HW * sizeof(unsigned long long), kWsAlign) : 0;
}

int small_bwd_launches(const Problem& p) { return p.g.shared ? 3 : 1; }

gspn_status small_fwd(const Problem& p, const DeviceInfo& dev, const void* x, const void* logits, const void* lam,
                      void* out, cudaStream_t s) {
    (void)dev;
    SmallArgs a{};
    a.g = p.g;
    a.x = x;
    a.logits = logits;
    a.lam = lam;
    a.out = out;
    const bool f32 = p.d.dtype == GSPN_F32, one = (p.g.H > p.g.W ? p.g.H : p.g.W) <= 32;
    // one position per lane when every line fits in 32 lanes: half the registers
    const void* fn = f32 ? (one ? (const void*)small_fwd_kernel<float, 1> : (const void*)small_fwd_kernel<float, 2>)
                         : (one ? (const void*)small_fwd_kernel<__nv_bfloat16, 1>
                                : (const void*)small_fwd_kernel<__nv_bfloat16, 2>);
    const int smem = (int)fwd_smem(p);
    if (ensure_smem_attr(fn, smem, (f32 ? 22 : 23) + (one ? 4 : 0)) != cudaSuccess) return GSPN_ERR_CUDA;
    void* args[] = {&a};
    if (cudaLaunchKernel(fn, dim3((unsigned)p.planes), dim3(32 * p.g.D), args, smem, s) != cudaSuccess)
        return GSPN_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? GSPN_OK : GSPN_ERR_CUDA;
}

gspn_status small_bwd(const Problem& p, const DeviceInfo& dev, const void* x, const void* logits, const void* lam,
                      const void* dout, void* dx, void* dlogits, void* dlam, void* ws, cudaStream_t s) {
    (void)dev;
    SmallArgs a{};
    a.g = p.g;
    a.x = x;
    a.logits = logits;
    a.lam = lam;
    a.dout = dout;
    a.dx = dx;
    a.dlogits = dlogits;
    a.dlam = dlam;
    a.dlog_ws = static_cast<unsigned long long*>(ws);
    const int64_t nlog = (int64_t)p.g.D * p.g.B * 3 * p.HW;
    if (p.g.shared) {
        small_zero_kernel<<<grid_1d(nlog), 256, 0, s>>>(a.dlog_ws, nlog);
        if (cudaGetLastError() != cudaSuccess) return GSPN_ERR_CUDA;
    }
    const bool f32 = p.d.dtype == GSPN_F32, one = (p.g.H > p.g.W ? p.g.H : p.g.W) <= 32;
    const void* fn = f32 ? (one ? (const void*)small_bwd_kernel<float, 1> : (const void*)small_bwd_kernel<float, 2>)
                         : (one ? (const void*)small_bwd_kernel<__nv_bfloat16, 1>
                                : (const void*)small_bwd_kernel<__nv_bfloat16, 2>);
    const int smem = (int)bwd_smem(p);
    if (ensure_smem_attr(fn, smem, (f32 ? 24 : 25) + (one ? 4 : 0)) != cudaSuccess) return GSPN_ERR_CUDA;
    void* args[] = {&a};
    if (cudaLaunchKernel(fn, dim3((unsigned)p.planes), dim3(32 * p.g.D), args, smem, s) != cudaSuccess)
        return GSPN_ERR_CUDA;
    if (p.g.shared) {
        if (f32)
            small_convert_kernel<float><<<grid_1d(nlog), 256, 0, s>>>(a.dlog_ws, static_cast<float*>(dlogits), nlog);
        else
            small_convert_kernel<__nv_bfloat16>
                <<<grid_1d(nlog), 256, 0, s>>>(a.dlog_ws, static_cast<__nv_bfloat16*>(dlogits), nlog);
        if (cudaGetLastError() != cudaSuccess) return GSPN_ERR_CUDA;
    }
    return GSPN_OK;
}

}  // namespace gspn
