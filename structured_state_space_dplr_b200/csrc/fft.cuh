// fft.cuh -- shared-memory mixed-radix FFT building blocks for sm_100a.
//
// A CTA holds m = 2^LG complex points in shared memory and transforms them
// in place with radix-16 first and last passes and the bits left over in
// the fewest middle passes of radix at most 32, each thread keeping a whole
// radix group in registers:
//
//   forward  = decimation in frequency: natural input -> digit-reversed
//              output (no reorder pass);
//   inverse  = decimation in time: digit-reversed input -> natural output.
//
// So a convolution needs no permutation at all: transform, multiply by a
// spectrum stored in the same digit-reversed order, transform back. The last
// forward pass and the first inverse pass touch the same groups of R
// consecutive points, so they are fused with the pointwise product and the
// data stays in registers across them.
//
// A length-N transform is split over C ranks (N = C m): rank c owns the
// frequencies C f + c and transforms its own input
//     v_c[k] = W_N^{k c} sum_r x[k + r m] W_C^{r c};
// inverse, each rank runs an m-point transform and the C partial results are
// combined:
//     x[k + r m] = sum_c W_C^{-c r} W_N^{-c k} Z_c[k].
// The twist W_N^{k c} is folded into the first pass: a per-rank constant on
// each input of a group (pre) and, with the pass twiddles, ta[j] tb[j]^q
// formed by recurrence from two tables of m/16 entries (build_rank_tables).
//
// Shared memory is padded by two points after every 16 (pidx below): with
// the pass plan, every pass is free of bank conflicts.
#pragma once
#include "common.cuh"

namespace s4 {

// ------------------------------------------------------------------ plan --
// log2 of the radix of pass s for a 2^lg-point transform. The last pass is
// radix 16 and so is the first (radix 32 from lg = 14 on); the bits left
// over go to the fewest middle passes of radix at most 32, split as evenly
// as they allow (lg = 13: 16 x 32 x 16, lg = 14: 32 x 32 x 16, three passes;
// every pass is one round trip through shared memory, which bounds these
// transforms as much as the arithmetic does). Every strided pass then has a stride of at least 16 points and the
// last pass works on 16 consecutive points (moved as 16-byte pairs), which
// keeps all of them free of shared-memory bank conflicts with the padding
// below.
// radix bits of the first pass: 16, or 32 from 2^14 points on (one middle
// pass of radix 32 then still covers the rest)
__host__ __device__ constexpr int plan_first(int lg) { return lg >= 14 ? 5 : 4; }
__host__ __device__ constexpr int plan_P(int lg) { return lg <= 8 ? 2 : 2 + (lg - plan_first(lg) - 4 + 4) / 5; }
__host__ __device__ constexpr int plan_lr(int lg, int s) {
    if (lg == 4) return 2;
    if (lg <= 8) return s == 0 ? lg - 4 : 4;
    if (s == 0) return plan_first(lg);
    if (s == plan_P(lg) - 1) return 4;
    const int k = plan_P(lg) - 2, mid = lg - plan_first(lg) - 4;
    return mid / k + (s - 1 < mid % k ? 1 : 0);
}
// block size of pass s (the sub-transform length it starts)
__host__ __device__ constexpr int plan_B(int lg, int s) {
    int b = lg;
    for (int i = 0; i < s; ++i) b -= plan_lr(lg, i);
    return 1 << b;
}
// Middle passes 1 .. P-2 keep one base twiddle W_B^j per group index j
// (S_s entries for pass s); the powers W_B^{j q} follow by a recurrence.
// Offset of pass s's base table (pass 0 has its own tables):
__host__ __device__ constexpr int plan_tw_off(int lg, int s) {
    int o = 0;
    for (int i = 1; i < s; ++i) o += plan_B(lg, i) >> plan_lr(lg, i);
    return o;
}
// all base twiddles of passes 1 .. P-2 (the last pass has none)
__host__ __device__ constexpr int plan_tw_size(int lg) { return plan_tw_off(lg, plan_P(lg) - 1); }

// Shared-memory padding: two points after every 16. Groups of the strided
// passes stay conflict-free for 8-byte accesses, and the contiguous groups of
// the last pass start on 16-byte boundaries, so they move as 16-byte vectors.
__host__ __device__ constexpr int padded(int m) { return m + m / 8; }
__device__ __forceinline__ int pidx(int i) { return i + 2 * (i >> 4); }

// frequency index held at position p after the forward passes
template <int LG>
__device__ __forceinline__ int digrev(int p) {
    int f = 0;
    static_for<0, plan_P(LG)>([&](auto sc) {
        constexpr int s = decltype(sc)::value;
        constexpr int lr = plan_lr(LG, s);
        constexpr int lS = ilog2(plan_B(LG, s)) - lr;            // log2 stride
        constexpr int lw = LG - ilog2(plan_B(LG, s));            // log2(m / B)
        f |= ((p >> lS) & ((1 << lr) - 1)) << lw;
    });
    return f;
}

// position holding frequency f after the forward passes (inverse of digrev)
template <int LG>
__device__ __forceinline__ int digrev_inv(int f) {
    int p = 0;
    static_for<0, plan_P(LG)>([&](auto sc) {
        constexpr int s = decltype(sc)::value;
        constexpr int lr = plan_lr(LG, s);
        constexpr int lS = ilog2(plan_B(LG, s)) - lr;
        constexpr int lw = LG - ilog2(plan_B(LG, s));
        p |= ((f >> lw) & ((1 << lr) - 1)) << lS;
    });
    return p;
}

// ------------------------------------------------------------ butterflies --
// cos(2 pi e / 64) for any integer e (values of cos(k pi / 32), k = 0..16)
__host__ __device__ constexpr float cos64(int e) {
    constexpr float c[17] = {1.0f, 0.99518472667219693f, 0.98078528040323043f, 0.95694033573220882f,
                             0.92387953251128674f, 0.88192126434835505f, 0.83146961230254524f,
                             0.77301045336273699f, 0.70710678118654752f, 0.63439328416364549f,
                             0.55557023301960218f, 0.47139673682599781f, 0.38268343236508977f,
                             0.29028467725446233f, 0.19509032201612827f, 0.09801714032956077f, 0.0f};
    const int k = ((e % 64) + 64) % 64;          // angle k pi / 32 in [0, 2 pi)
    return k <= 16 ? c[k] : (k <= 32 ? -c[32 - k] : (k <= 48 ? -c[k - 32] : c[64 - k]));
}
__host__ __device__ constexpr float sin64(int e) { return cos64(e - 16); }

// v * exp(DIR * 2 pi i E / N), N in {2, 4, 8, 16, 32, 64}
template <int E, int N, int DIR>
__device__ __forceinline__ float2 rot(float2 v) {
    static_assert(N >= 2 && N <= 64 && (N & (N - 1)) == 0, "rot: N a power of two up to 64");
    constexpr int e = ((E * (64 / N)) % 64 + 64) % 64;
    if constexpr (e == 0) return v;
    else if constexpr (e == 16) return mul_i<DIR>(v);
    else if constexpr (e == 32) return make_float2(-v.x, -v.y);
    else if constexpr (e == 48) return mul_i<-DIR>(v);
    else {
        constexpr float c = cos64(e);
        constexpr float s = DIR > 0 ? sin64(e) : -sin64(e);
        if constexpr (e % 8 == 0) {  // (+-1 +- i)/sqrt(2)
            constexpr float h = 0.70710678118654752f;
            constexpr float sc = c > 0 ? 1.0f : -1.0f, ss = s > 0 ? 1.0f : -1.0f;
            float re = sc * v.x - ss * v.y, im = ss * v.x + sc * v.y;
            return make_float2(h * re, h * im);
        } else {
            return make_float2(fmaf(v.x, c, -v.y * s), fmaf(v.x, s, v.y * c));
        }
    }
}

template <int DIR>
__device__ __forceinline__ void dft4(float2 &x0, float2 &x1, float2 &x2, float2 &x3) {
    float2 a0 = cadd(x0, x2), a1 = csub(x0, x2), a2 = cadd(x1, x3), a3 = mul_i<DIR>(csub(x1, x3));
    x0 = cadd(a0, a2); x2 = csub(a0, a2); x1 = cadd(a1, a3); x3 = csub(a1, a3);
}

// in-register DFT of length R (natural order in and out), kernel exp(DIR 2 pi i n k / R)
template <int R, int DIR>
__device__ __forceinline__ void dft(float2 (&x)[R]) {
    if constexpr (R == 2) {
        float2 a = x[0]; x[0] = cadd(a, x[1]); x[1] = csub(a, x[1]);
    } else if constexpr (R == 4) {
        dft4<DIR>(x[0], x[1], x[2], x[3]);
    } else {
        constexpr int R2 = R / 4;   // n = R2 n1 + n2, k = k1 + 4 k2
        float2 y[R];
        static_for<0, R2>([&](auto n2c) {
            constexpr int n2 = decltype(n2c)::value;
            float2 a0 = x[n2], a1 = x[R2 + n2], a2 = x[2 * R2 + n2], a3 = x[3 * R2 + n2];
            dft4<DIR>(a0, a1, a2, a3);
            y[n2 * 4 + 0] = a0;
            y[n2 * 4 + 1] = rot<n2 * 1, R, DIR>(a1);
            y[n2 * 4 + 2] = rot<n2 * 2, R, DIR>(a2);
            y[n2 * 4 + 3] = rot<n2 * 3, R, DIR>(a3);
        });
        static_for<0, 4>([&](auto k1c) {
            constexpr int k1 = decltype(k1c)::value;
            float2 b[R2];
            static_for<0, R2>([&](auto n2c) { b[decltype(n2c)::value] = y[decltype(n2c)::value * 4 + k1]; });
            dft<R2, DIR>(b);
            static_for<0, R2>([&](auto k2c) { x[k1 + 4 * decltype(k2c)::value] = b[decltype(k2c)::value]; });
        });
    }
}

// ---------------------------------------------------------------- tables --
// Base twiddles of the middle passes: tws[off_s + j] = W_{B_s}^j, j < S_s.
template <int LG>
__device__ void build_middle_tables(float2 *tws, int tid, int nthreads) {
    static_for<1, plan_P(LG) - 1>([&](auto sc) {
        constexpr int s = decltype(sc)::value;
        constexpr int B = plan_B(LG, s);
        constexpr int S = B >> plan_lr(LG, s);
        float2 *t = tws + plan_tw_off(LG, s);
        for (int j = tid; j < S; j += nthreads) t[j] = unit_root(j, B);
    });
}

// ---------------------------------------------------------------- passes --
// In every pass, group member q sits at padded index pidx(base) + off(q S):
// (base mod 16) + (q S mod 16) < 16 holds for all plans, so the padding term
// of base + q S splits into that of base plus (q S) / 16 -- a constant.
template <int QS>
__host__ __device__ constexpr int poff() { return QS + 2 * (QS >> 4); }

// R consecutive points starting at a 16-byte aligned shared address
template <int R>
__device__ __forceinline__ void load_contig(const float2 *p, float2 (&x)[R]) {
    static_for<0, R / 2>([&](auto i) {
        const float4 v = reinterpret_cast<const float4 *>(p)[i];
        x[2 * i] = make_float2(v.x, v.y);
        x[2 * i + 1] = make_float2(v.z, v.w);
    });
}
template <int R>
__device__ __forceinline__ void store_contig(float2 *p, const float2 (&x)[R]) {
    static_for<0, R / 2>([&](auto i) {
        reinterpret_cast<float4 *>(p)[i] = make_float4(x[2 * i].x, x[2 * i].y, x[2 * i + 1].x, x[2 * i + 1].y);
    });
}
// x[q] *= w^q (q >= 1) with the powers of w formed on the fly
template <int DIR, int R>
__device__ __forceinline__ void apply_powers(float2 (&x)[R], float2 w) {
    float2 wq = w;
    static_for<1, R>([&](auto q) {
        x[q] = ctw<DIR>(x[q], wq);
        if constexpr (decltype(q)::value + 1 < R) wq = cmul(wq, w);
    });
}
template <int DIR, int R>
__device__ __forceinline__ void apply_powers2(float2 (&x)[R], float2 (&z)[R], float2 w) {
    float2 wq = w;
    static_for<1, R>([&](auto q) {
        x[q] = ctw<DIR>(x[q], wq);
        z[q] = ctw<DIR>(z[q], wq);
        if constexpr (decltype(q)::value + 1 < R) wq = cmul(wq, w);
    });
}

// Middle pass s (1 <= s <= P-1) in decimation-in-frequency form: DFT of each
// group, then twiddles. DIR = -1 forward, +1 inverse (conjugate twiddles).
template <int LG, int s, int DIR, int T>
__device__ __forceinline__ void dif_pass(float2 *buf, const float2 *tws, int tid = threadIdx.x) {
    constexpr int lr = plan_lr(LG, s), R = 1 << lr;
    constexpr int B = plan_B(LG, s), S = B / R, G = (1 << LG) / R;
    constexpr int lS = ilog2(S);
    const float2 *tw = tws + plan_tw_off(LG, s);
    for (int g = tid; g < G; g += T) {
        const int j = g & (S - 1);
        float2 *p = buf + pidx(((g >> lS) << (lS + lr)) + j);
        float2 x[R];
        if constexpr (S == 1) load_contig<R>(p, x);
        else static_for<0, R>([&](auto q) { x[q] = p[poff<decltype(q)::value * S>()]; });
        dft<R, DIR>(x);
        if constexpr (S > 1) apply_powers<DIR, R>(x, tw[j]);
        if constexpr (S == 1) store_contig<R>(p, x);
        else static_for<0, R>([&](auto q) { p[poff<decltype(q)::value * S>()] = x[q]; });
    }
}

// Middle pass s in decimation-in-time form (the transpose): twiddles, then DFT.
template <int LG, int s, int DIR, int T>
__device__ __forceinline__ void dit_pass(float2 *buf, const float2 *tws, int tid = threadIdx.x) {
    constexpr int lr = plan_lr(LG, s), R = 1 << lr;
    constexpr int B = plan_B(LG, s), S = B / R, G = (1 << LG) / R;
    constexpr int lS = ilog2(S);
    const float2 *tw = tws + plan_tw_off(LG, s);
    for (int g = tid; g < G; g += T) {
        const int j = g & (S - 1);
        float2 *p = buf + pidx(((g >> lS) << (lS + lr)) + j);
        float2 x[R];
        if constexpr (S == 1) load_contig<R>(p, x);
        else static_for<0, R>([&](auto q) { x[q] = p[poff<decltype(q)::value * S>()]; });
        if constexpr (S > 1) apply_powers<DIR, R>(x, tw[j]);
        dft<R, DIR>(x);
        if constexpr (S == 1) store_contig<R>(p, x);
        else static_for<0, R>([&](auto q) { p[poff<decltype(q)::value * S>()] = x[q]; });
    }
}

// Forward passes 1 .. P-2 (pass 0 and the last pass are done by the caller).
template <int LG, int T>
__device__ __forceinline__ void forward_middle(float2 *buf, const float2 *tws, int tid = threadIdx.x) {
    static_for<1, plan_P(LG) - 1>([&](auto sc) {
        dif_pass<LG, decltype(sc)::value, -1, T>(buf, tws, tid);
        __syncthreads();
    });
}
// Inverse passes P-2 .. 1.
template <int LG, int T>
__device__ __forceinline__ void inverse_middle(float2 *buf, const float2 *tws, int tid = threadIdx.x) {
    constexpr int P = plan_P(LG);
    static_for<1, P - 1>([&](auto sc) {
        dit_pass<LG, P - 1 - decltype(sc)::value, +1, T>(buf, tws, tid);
        __syncthreads();
    });
}

// Per-CTA tables of rank c of a C-way split of an N = C m transform, small
// enough to sit in shared memory at every length: the first-pass twiddle
// W_N^{j (C q + c)} = W_N^{j c} W_m^{j q} is ta[j] tb[j]^q (j < S0, formed by
// recurrence over q), and pre[p] = W_{C R0}^{p c} is the in-group share of the
// rank's twist.
template <int LG>
__device__ void build_rank_tables(float2 *ta, float2 *tb, float2 *pre, int C, int c, int tid, int nthreads) {
    constexpr int m = 1 << LG;
    constexpr int R0 = 1 << plan_lr(LG, 0), S0 = m / R0;
    const int N = C * m;
    for (int j = tid; j < S0; j += nthreads) {
        ta[j] = unit_root((j * c) & (N - 1), N);
        tb[j] = unit_root(j, m);
    }
    for (int p = tid; p < R0; p += nthreads) pre[p] = unit_root((p * c) % (C * R0), C * R0);
}

// First forward pass of group j with the rank tables: x_p = fetch(j + p S0)
// pre[p], DFT, times ta[j] tb[j]^q.
template <int LG, class Fetch>
__device__ __forceinline__ void first_group_rec(float2 (&x)[1 << plan_lr(LG, 0)], int j, const float2 *ta,
                                                const float2 *tb, const float2 *pre, Fetch &&fetch) {
    constexpr int R = 1 << plan_lr(LG, 0);
    constexpr int S = (1 << LG) / R;
    static_for<0, R>([&](auto p) {
        const float2 v = fetch(j + p * S);
        if constexpr (decltype(p)::value == 0) x[p] = v; else x[p] = cmul(v, pre[p]);
    });
    dft<R, -1>(x);
    const float2 b = tb[j];
    float2 w = ta[j];
    static_for<0, R>([&](auto q) {
        x[q] = cmul(x[q], w);
        if constexpr (decltype(q)::value + 1 < R) w = cmul(w, b);
    });
}

// Last inverse pass with the rank tables (the conjugate of the above):
// W_N^{-c k} Z_c[k] stored at pidx(k), natural order.
template <int LG, int T>
__device__ __forceinline__ void inverse_last_rec(float2 *buf, const float2 *ta, const float2 *tb, const float2 *pre) {
    constexpr int R = 1 << plan_lr(LG, 0);
    constexpr int S = (1 << LG) / R;
    for (int j = threadIdx.x; j < S; j += T) {
        float2 *p = buf + pidx(j);
        const float2 b = tb[j];
        float2 w = ta[j];
        float2 x[R];
        static_for<0, R>([&](auto q) {
            x[q] = cmulc(p[poff<decltype(q)::value * S>()], w);
            if constexpr (decltype(q)::value + 1 < R) w = cmul(w, b);
        });
        dft<R, +1>(x);
        static_for<0, R>([&](auto q) {
            if constexpr (decltype(q)::value == 0) p[0] = x[q];
            else p[poff<decltype(q)::value * S>()] = cmulc(x[q], pre[q]);
        });
    }
}

template <int LG>
__device__ __forceinline__ void store_first_group(float2 *buf, const float2 (&x)[1 << plan_lr(LG, 0)], int j) {
    constexpr int R = 1 << plan_lr(LG, 0);
    constexpr int S = (1 << LG) / R;
    float2 *p = buf + pidx(j);
    static_for<0, R>([&](auto q) { p[poff<decltype(q)::value * S>()] = x[q]; });
}

// Fused last forward pass + pointwise product + first inverse pass. The group
// of R consecutive positions [g R, g R + R) is multiplied by mul(pos0, x);
// pre(pos0) runs first (to start loads early).
template <int LG, int T, class Mul>
__device__ __forceinline__ void fused_middle(float2 *buf, Mul &&mul, int tid = threadIdx.x) {
    constexpr int lr = plan_lr(LG, plan_P(LG) - 1), R = 1 << lr;
    constexpr int G = (1 << LG) / R;
    for (int g = tid; g < G; g += T) {
        const int base = g * R;
        float2 *p = buf + pidx(base);
        float2 x[R];
        load_contig<R>(p, x);
        dft<R, -1>(x);
        mul(base, x);
        dft<R, +1>(x);
        store_contig<R>(p, x);
    }
}

// Last forward pass only, handing each finished group to out(pos0, x).
template <int LG, int T, class Out>
__device__ __forceinline__ void forward_last(float2 *buf, Out &&out) {
    constexpr int lr = plan_lr(LG, plan_P(LG) - 1), R = 1 << lr;
    constexpr int G = (1 << LG) / R;
    for (int g = threadIdx.x; g < G; g += T) {
        const int base = g * R;
        const float2 *p = buf + pidx(base);
        float2 x[R];
        load_contig<R>(p, x);
        dft<R, -1>(x);
        out(base, x);
    }
}

// Storage of a spectrum produced by the last forward pass (one channel and
// rank): group g of that pass holds the R consecutive positions
// [g R, g R + R), kept as R/2 float4 words. Word i of every group is stored
// contiguously (index i G + g, G = m / R), so the consecutive threads of a
// warp, which own consecutive groups, read and write consecutive words.
template <int LG>
__device__ __forceinline__ int spec4_index(int base, int i) {
    constexpr int R = 1 << plan_lr(LG, plan_P(LG) - 1);
    constexpr int G = (1 << LG) / R;
    return i * G + base / R;
}

// Gather the input of an inverse transform into digit-reversed positions:
// frequency f goes to the position that holds it. Threads take consecutive
// frequencies, so value(f) may read global memory in order (coalesced); the
// scattered side is the shared-memory store.
template <int LG, int T, class Val>
__device__ __forceinline__ void gather_digit_reversed(float2 *buf, Val &&value) {
    for (int f = threadIdx.x; f < (1 << LG); f += T) buf[pidx(digrev_inv<LG>(f))] = value(f);
}

// ------------------------------------------------- two transforms at once --
// The same pass applied to the same group of two independent buffers by one
// thread: twice the independent work per thread (the two halves of a
// length-2m transform, see k_fftconv_pair).
template <int LG, int s, int DIR, bool TW_FIRST, int T>
__device__ __forceinline__ void pass_x2(float2 *b0, float2 *b1, const float2 *tws) {
    constexpr int lr = plan_lr(LG, s), R = 1 << lr;
    constexpr int B = plan_B(LG, s), S = B / R, G = (1 << LG) / R;
    constexpr int lS = ilog2(S);
    const float2 *tw = tws + plan_tw_off(LG, s);
    if constexpr (R >= 32) {
        // a group of both buffers would hold 2R points in registers: each
        // thread takes one group of one buffer instead (2G groups in all)
        for (int i = threadIdx.x; i < 2 * G; i += T) {
            float2 *b = i < G ? b0 : b1;
            const int g = i < G ? i : i - G;
            const int j = g & (S - 1);
            float2 *p = b + pidx(((g >> lS) << (lS + lr)) + j);
            float2 x[R];
            static_for<0, R>([&](auto q) { x[q] = p[poff<decltype(q)::value * S>()]; });
            if constexpr (TW_FIRST) apply_powers<DIR, R>(x, tw[j]);
            dft<R, DIR>(x);
            if constexpr (!TW_FIRST) apply_powers<DIR, R>(x, tw[j]);
            static_for<0, R>([&](auto q) { p[poff<decltype(q)::value * S>()] = x[q]; });
        }
        return;
    }
    for (int g = threadIdx.x; g < G; g += T) {
        const int j = g & (S - 1);
        const int o = pidx(((g >> lS) << (lS + lr)) + j);
        float2 x[R], z[R];
        if constexpr (S == 1) {
            load_contig<R>(b0 + o, x);
            load_contig<R>(b1 + o, z);
        } else {
            static_for<0, R>([&](auto q) {
                x[q] = b0[o + poff<decltype(q)::value * S>()];
                z[q] = b1[o + poff<decltype(q)::value * S>()];
            });
        }
        if constexpr (TW_FIRST && S > 1) apply_powers2<DIR, R>(x, z, tw[j]);
        dft<R, DIR>(x);
        dft<R, DIR>(z);
        if constexpr (!TW_FIRST && S > 1) apply_powers2<DIR, R>(x, z, tw[j]);
        if constexpr (S == 1) {
            store_contig<R>(b0 + o, x);
            store_contig<R>(b1 + o, z);
        } else {
            static_for<0, R>([&](auto q) {
                b0[o + poff<decltype(q)::value * S>()] = x[q];
                b1[o + poff<decltype(q)::value * S>()] = z[q];
            });
        }
    }
}
template <int LG, int T>
__device__ __forceinline__ void forward_middle_x2(float2 *b0, float2 *b1, const float2 *tws) {
    static_for<1, plan_P(LG) - 1>([&](auto sc) {
        pass_x2<LG, decltype(sc)::value, -1, false, T>(b0, b1, tws);
        __syncthreads();
    });
}
template <int LG, int T>
__device__ __forceinline__ void inverse_middle_x2(float2 *b0, float2 *b1, const float2 *tws) {
    constexpr int P = plan_P(LG);
    static_for<1, P - 1>([&](auto sc) {
        pass_x2<LG, P - 1 - decltype(sc)::value, +1, true, T>(b0, b1, tws);
        __syncthreads();
    });
}
// last forward pass, product with the two spectra (mul(pos0, x, z)), first
// inverse pass, for both buffers
template <int LG, int T, class Fetch, class Mul>
__device__ __forceinline__ void fused_middle_x2(float2 *b0, float2 *b1, Fetch &&fetch, Mul &&mul) {
    constexpr int lr = plan_lr(LG, plan_P(LG) - 1), R = 1 << lr;
    constexpr int G = (1 << LG) / R;
    for (int g = threadIdx.x; g < G; g += T) {
        const int base = g * R;
        const int o = pidx(base);
        auto spec = fetch(base);   // issued before the transforms that hide its latency
        float2 x[R], z[R];
        load_contig<R>(b0 + o, x);
        load_contig<R>(b1 + o, z);
        dft<R, -1>(x);
        dft<R, -1>(z);
        mul(spec, x, z);
        dft<R, +1>(x);
        dft<R, +1>(z);
        store_contig<R>(b0 + o, x);
        store_contig<R>(b1 + o, z);
    }
}

// ------------------------------------------- warp-level middle barriers --
// With a single middle pass of radix R1, that pass hands each block of
// B1 = m / R0 points to S1 = B1 / R1 consecutive threads. When the fused pass
// (last forward pass, product, first inverse pass) takes a block's groups
// with the same threads, nothing written in one of these three passes is read
// by another warp in the next, and the barriers between them are __syncwarp.
// Two layouts qualify (R0 = RL = 16, one middle-pass item per thread):
//   16 x 16 x 16, two buffers, T = m / 16: thread g runs group g of both
//     buffers in every pass (fused_middle_x2 already does), S1 = 16;
//   16 x 32 x 16, T = m / 16 on two buffers (thread i: buffer i / (m/32)) or
//     T = m / 32 on one: the radix-32 pass gives thread t the block
//     (t % (m/32)) / 16 of its buffer, and fused_blocks(_x2) give it that
//     block's 16-point groups (t % 16) and (t % 16) + 16.
template <int LG, int T, int NBUF>
__host__ __device__ constexpr bool warp_local_middle() {
    return plan_P(LG) == 3 && plan_lr(LG, 0) == 4 && plan_lr(LG, 2) == 4 &&
           ((plan_lr(LG, 1) == 4 && NBUF == 2 && T == (1 << LG) / 16) ||
            (plan_lr(LG, 1) == 5 && T == NBUF * ((1 << LG) / 32)));
}

// the fused pass of the 16 x 32 x 16 plan, one buffer or two, spectrum words
// in spec4_index order from kp (buffer b0 / the single buffer) and kq (b1)
template <int LG, int NBUF, bool CONJ>
__device__ __forceinline__ void fused_blocks(float2 *b0, float2 *b1, const float4 *__restrict__ kp,
                                             const float4 *__restrict__ kq) {
    constexpr int R = 16, GM = (1 << LG) / 32;   // radix-32 groups per buffer
    static_assert(plan_lr(LG, 1) == 5 && plan_lr(LG, 2) == 4, "the 16 x 32 x 16 plan");
    const int i = threadIdx.x;
    const bool second = NBUF == 2 && i >= GM;
    float2 *b = second ? b1 : b0;
    const float4 *k = second ? kq : kp;
    const int t = i % GM;
    const int g0 = (t >> 4) * 32 + (t & 15), g1 = g0 + 16;
    float4 w0[R / 2], w1[R / 2];
    static_for<0, R / 2>([&](auto ii) {
        w0[ii] = __ldg(k + spec4_index<LG>(g0 * R, ii));
        w1[ii] = __ldg(k + spec4_index<LG>(g1 * R, ii));
    });
    float2 x[R], z[R];
    load_contig<R>(b + pidx(g0 * R), x);
    load_contig<R>(b + pidx(g1 * R), z);
    dft<R, -1>(x);
    dft<R, -1>(z);
    auto mul = [](float2 a, float x0, float x1) {
        if constexpr (CONJ) return cmulc(a, make_float2(x0, x1)); else return cmul(a, make_float2(x0, x1));
    };
    static_for<0, R / 2>([&](auto ii) {
        x[2 * ii] = mul(x[2 * ii], w0[ii].x, w0[ii].y);
        x[2 * ii + 1] = mul(x[2 * ii + 1], w0[ii].z, w0[ii].w);
        z[2 * ii] = mul(z[2 * ii], w1[ii].x, w1[ii].y);
        z[2 * ii + 1] = mul(z[2 * ii + 1], w1[ii].z, w1[ii].w);
    });
    dft<R, +1>(x);
    dft<R, +1>(z);
    store_contig<R>(b + pidx(g0 * R), x);
    store_contig<R>(b + pidx(g1 * R), z);
}

}  // namespace s4
