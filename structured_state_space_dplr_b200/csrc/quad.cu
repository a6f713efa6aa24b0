// quad.cu -- the convolution at L = 16384 and the spectra it reads
// ("The S4 kernel, from scratch", §4 kernel via the generating function and
// its inverse FFT, §5 fft_conv): the zero-padded length-2L transform split
// four ways over a cluster of two CTAs, each holding two ranks as the two
// halves of the one-CTA pair kernel (pairs.cuh).
//
// k_fftconv_quad    : the convolution, persistent over row pairs;
// k_kspec_quad      : the spectrum of K + D delta_0 from K (or K + i Ki);
// k_kspec_quad_half : the same from k_cauchy's packed half spectrum, with the
//                     inverse real transform folded in (K stored in place).
#include <cooperative_groups.h>

#include "cluster.cuh"
#include "fft.cuh"
#include "launch.h"
#include "pairs.cuh"

namespace cg = cooperative_groups;

namespace s4 {

// a hint that brings the line holding p into L2 (no registers, no completion)
__device__ __forceinline__ void l2_prefetch(const void *p) {
    asm volatile("prefetch.global.L2 [%0];" ::"l"(__cvta_generic_to_global(p)));
}

// ------------------------------------------------ fftconv, cluster of two --
// L = 16384: the zero-padded length-N = 2L transform split four ways, rank c
// holding the frequencies 4f + c (m = N/4 = 8192 points each). With the
// nonzero input in two chunks x0[k] = x[k], x1[k] = x[k + m] (k < m), rank c
// transforms v_c[k] = W_N^{kc} (x0[k] + (-i)^c x1[k]), and the output points
// k and k + m are
//   x[k + r m] = sum_c i^{c r} W_N^{-ck} Z_c[k]     (Z_c: rank c after the
//                                                    product and the inverse).
// A cluster of two CTAs takes a row pair; CTA 0 holds ranks 0 and 2, CTA 1
// ranks 1 and 3, as the two halves of the one-CTA kernel (rank c + 2 is rank
// c twisted by W_N^{2k} = W_2m^k, the halves' relation there):
//   CTA 0: halves from x0 + x1 and x0 - x1;
//   CTA 1: halves from W_N^k (x0 - i x1) and W_N^k (x0 + i x1).
// The halves' last inverse pass gives each CTA their sum S and difference M
// at every k, and
//   x[k] = S_0 + W_N^-k S_1,   x[k + m] = M_0 + i W_N^-k M_1.
// So CTA 0 keeps S_0 and hands M_0 over, CTA 1 keeps i W_N^-k M_1 and hands
// W_N^-k S_1 over; CTA 0 writes x[k], CTA 1 x[k + m]. The kept values stay in
// the CTA's own buffer and the hand-over goes into the partner's receive
// buffer with distributed-shared-memory stores (which do not wait on a round
// trip), under a split cluster barrier: release after the stores, acquire
// before reading the own buffer, and a relaxed arrive once it is read, which
// the partner waits on before its next stores. The spectrum holds 4 ranks x
// m points per channel (k_kspec_quad).
constexpr int kQuadLG = 13;

// the two ranks' inputs of point k = j + p S0 from the chunks a = x0[k], b = x1[k]
template <int P>
__device__ __forceinline__ void quad_inputs(int cr, float2 a, float2 b, float2 &v0, float2 &v1) {
    if (cr == 0) {
        v0 = cadd(a, b);
        v1 = csub(a, b);
    } else {   // W_N^{p S0} = W_64^p inside the group; W_N^j goes with the group twiddles
        v0 = rot<P, 64, -1>(cadd(a, mul_i<-1>(b)));
        v1 = rot<P, 64, -1>(cadd(a, mul_i<+1>(b)));
    }
}

template <bool CONJ>
__global__ void __launch_bounds__(pair_threads<kQuadLG>(), 1)
k_fftconv_quad(const float *__restrict__ u, const float2 *__restrict__ spec, int Bt, int H, float *__restrict__ y) {
    constexpr int LG = kQuadLG, m = 1 << LG, L = 2 * m, T = pair_threads<LG>();
    constexpr int R0 = 1 << plan_lr(LG, 0), S0 = m / R0;
    constexpr int RL = 1 << plan_lr(LG, plan_P(LG) - 1);
    static_assert(S0 == T, "one first-pass group per thread");
    extern __shared__ float2 sm[];
    const PairSmem s = pair_carve<LG>(sm);
    // the partner's hand-over lands in this CTA's stage area (m points, one
    // per (thread, p): index t = j + p S0), written there by the partner with
    // remote stores, so the exchange never waits on a remote load
    float2 *recv = reinterpret_cast<float2 *>(s.stage);
    cg::cluster_group cluster = cg::this_cluster();
    const int cr = (int)cluster.block_rank();
    float2 *precv = cluster.map_shared_rank(recv, cr ^ 1);
    pair_tables<LG>(s);
    const int j = threadIdx.x;
    const float2 tcj = unit_root(j, 2 * L);   // W_N^j
    const float2 cj = cconj(tcj);             // W_N^-j
    cluster.sync();   // both CTAs run before either reaches into the other's memory
    const long long npairs = (long long)H * ((Bt + 1) / 2);
    const long long cl = blockIdx.x / 2, ncl = gridDim.x / 2;
    // a[p], b[p]: the two input chunks (row 0 + i row 1) at k = j + p S0
    // (holding them a pair ahead, across the exchange, costs more in
    // registers than it hides in latency)
    float2 a[R0], b[R0];
    auto load_inputs = [&](long long pr) {
        const RowPair r = row_pair(pr, Bt);
        const float *u0 = u + ((size_t)r.b0 * H + r.h) * L;
        const float *u1 = u0 + (size_t)H * L;
        static_for<0, R0>([&](auto p) {
            const int k = j + p * S0;
            a[p] = make_float2(__ldg(u0 + k), r.has1 ? __ldg(u1 + k) : 0.0f);
            b[p] = make_float2(__ldg(u0 + k + m), r.has1 ? __ldg(u1 + k + m) : 0.0f);
        });
    };
    bool first = true;
    for (long long pr = cl; pr < npairs; pr += ncl) {
        const RowPair r = row_pair(pr, Bt);
        // the cluster's next row pair into L2 (CTA cr takes row cr, a 128-byte
        // line per thread), so its loads a pair from now hit L2 rather than
        // HBM: 251.8 -> 239.6 us at H = 256, batch 8. Two or three pairs ahead
        // was slower (247.9, 259.0 us), and so was also prefetching the next
        // channel's spectrum (245.7 us).
        if (pr + ncl < npairs) {
            const RowPair rn = row_pair(pr + ncl, Bt);
            if (cr == 0 || rn.has1) l2_prefetch(u + ((size_t)(rn.b0 + cr) * H + rn.h) * L + (size_t)j * 32);
        }
        load_inputs(pr);
        {
            float2 v0[R0], v1[R0];
            static_for<0, R0>([&](auto p) { quad_inputs<decltype(p)::value>(cr, a[p], b[p], v0[p], v1[p]); });
            if (cr == 0) first_pass_halves2<LG, false>(s, v0, v1, j, make_float2(1.0f, 0.0f));
            else first_pass_halves2<LG, true>(s, v0, v1, j, tcj);
        }
        __syncthreads();
        forward_middle_x2<LG, T>(s.b0, s.b1, s.tws);
        const float2 *sh = spec + (size_t)r.h * 2 * L;
        const float4 *k0p = reinterpret_cast<const float4 *>(sh + (size_t)cr * m);
        const float4 *k1p = reinterpret_cast<const float4 *>(sh + (size_t)(cr + 2) * m);
        struct SpecWords { float4 k0[RL / 2], k1[RL / 2]; };
        fused_middle_x2<LG, T>(s.b0, s.b1, [&](int base) {
            SpecWords w;
            static_for<0, RL / 2>([&](auto i) {
                w.k0[i] = __ldg(k0p + spec4_index<LG>(base, i));
                w.k1[i] = __ldg(k1p + spec4_index<LG>(base, i));
            });
            return w;
        }, [&](const SpecWords &w, auto &x, auto &z) {
            auto mul = [](float2 a, float x0, float x1) {
                if constexpr (CONJ) return cmulc(a, make_float2(x0, x1)); else return cmul(a, make_float2(x0, x1));
            };
            static_for<0, RL / 2>([&](auto i) {
                x[2 * i] = mul(x[2 * i], w.k0[i].x, w.k0[i].y);
                x[2 * i + 1] = mul(x[2 * i + 1], w.k0[i].z, w.k0[i].w);
                z[2 * i] = mul(z[2 * i], w.k1[i].x, w.k1[i].y);
                z[2 * i + 1] = mul(z[2 * i + 1], w.k1[i].z, w.k1[i].w);
            });
        });
        __syncthreads();
        inverse_middle_x2<LG, T>(s.b0, s.b1, s.tws);
        // ---- last pass: keep one of (S, M) in registers, store the other
        // into the partner's receive buffer (once the partner has read the
        // previous pair's hand-over from it)
        if (!first) cluster_wait();
        float2 *keep = s.b1;   // position pidx(t) of this thread's own group
        last_pass_halves_sum<LG>(s, [&](auto pc, int t, float2 S, float2 M) {
            constexpr int p = decltype(pc)::value;
            const int kp = pidx(t);
            if (cr == 0) {
                keep[kp] = S;
                precv[t] = M;
            } else {   // W_N^-t = W_N^-j W_64^-p
                keep[kp] = mul_i<+1>(rot<p, 64, +1>(cmul(M, cj)));
                precv[t] = rot<p, 64, +1>(cmul(S, cj));
            }
        });
        cluster_arrive_release();
        cluster_wait();
        float *y0 = y + ((size_t)r.b0 * H + r.h) * L + (cr == 0 ? 0 : m);
        float *y1 = y0 + (size_t)H * L;
        static_for<0, R0>([&](auto p) {
            const int t = j + p * S0;
            const float2 o = cadd(keep[pidx(t)], recv[t]);
            y0[t] = o.x;
            if (r.has1) y1[t] = o.y;
        });
        cluster_arrive_relaxed();   // done reading the receive buffer
        first = false;
    }
    if (!first) cluster_wait();   // pairs the last arrive
}

// The spectrum k_fftconv_quad reads: per channel 4 ranks x m points in
// spec4_index order, rank c holding (FFT_N(K + D delta_0))[4f + c] / N. One
// CTA per (channel, rank pair), persistent; K's two chunks enter as the
// convolution's input rows do.
template <bool CPLX>
__global__ void __launch_bounds__(pair_threads<kQuadLG>(), 1)
k_kspec_quad(const float *__restrict__ K, const float *__restrict__ Ki, const float *__restrict__ D, int H,
             float2 *__restrict__ spec) {
    constexpr int LG = kQuadLG, m = 1 << LG, L = 2 * m;
    constexpr int R0 = 1 << plan_lr(LG, 0), S0 = m / R0;
    extern __shared__ float2 sm[];
    const PairSmem s = pair_carve<LG>(sm);
    pair_tables<LG>(s);
    const int j = threadIdx.x;
    const float2 tcj = unit_root(j, 2 * L);   // W_N^j
    __syncthreads();
    for (int it = blockIdx.x; it < 2 * H; it += gridDim.x) {
        const int h = it >> 1, cr = it & 1;
        const float *Kh = K + (size_t)h * L;
        const float *Kih = CPLX ? Ki + (size_t)h * L : nullptr;
        float2 v0[R0], v1[R0];
        static_for<0, R0>([&](auto p) {
            const int k = j + p * S0;
            quad_inputs<decltype(p)::value>(cr, make_float2(__ldg(Kh + k), CPLX ? __ldg(Kih + k) : 0.0f),
                                           make_float2(__ldg(Kh + k + m), CPLX ? __ldg(Kih + k + m) : 0.0f),
                                           v0[p], v1[p]);
        });
        if (cr == 0) first_pass_halves2<LG, false>(s, v0, v1, j, make_float2(1.0f, 0.0f));
        else first_pass_halves2<LG, true>(s, v0, v1, j, tcj);
        __syncthreads();
        float4 *sh = reinterpret_cast<float4 *>(spec + (size_t)h * 2 * L);
        spectrum_tail2<LG>(s, D != nullptr ? __ldg(D + h) : 0.0f, 1.0f / (float)(2 * L), sh + (size_t)cr * (m / 2),
                           sh + (size_t)(cr + 2) * (m / 2));
        __syncthreads();
    }
}

// The same spectrum straight from the packed half spectrum that k_cauchy
// leaves in K (K[0] = K_hat_0, K[1] = K_hat_{L/2}, K[2f], K[2f+1] = K_hat_f,
// all times 1/L), with the inverse real transform folded in, so K does not
// round-trip through memory between the two: one cluster of two CTAs per
// channel, CTA cr holding ranks cr and cr + 2 as in k_kspec_quad. With
// M = L/2 and w = e^{2 pi i/L}, the length-M sequence
//   Z[k] = (X[k] + conj X[M-k]) + i w^k (X[k] - conj X[M-k])
// has the unnormalised inverse transform z[n] = K[2n] + i K[2n+1]. CTA cr
// inverts the frequencies k = 2k' + cr (a length-M/2 transform z_cr; Z[k]
// and Z[M-k] share a parity, so each pair of loads stays in one CTA), and
//   z[n] = z_0[n'] + e^{2 pi i n/M} z_1[n'],  n' = n mod M/2.
// The CTAs exchange z_cr through each other's stage area (distributed
// shared-memory stores, split cluster barrier as in k_fftconv_quad); then
// both read the chunks x0 = K[0, m), x1 = K[m, 2m) of the zero-padded
// transform: for k < m, K[k] and K[k + m] are components of
// z_0[k/2] +- e^{2 pi i (k/2)/M} z_1[k/2]. CTA 0 stores K[0, m) and CTA 1
// K[m, 2m) in place of the half spectrum; the barrier of the exchange orders
// those stores after both CTAs' reads of it.
__global__ void __launch_bounds__(pair_threads<kQuadLG>(), 1)
k_kspec_quad_half(float *__restrict__ K, const float *__restrict__ D, int H, float2 *__restrict__ spec) {
    constexpr int LG = kQuadLG, m = 1 << LG, L = 2 * m, M = L / 2, T = pair_threads<LG>();
    constexpr int LGH = LG - 1, MH = M / 2;                        // the half-length inverse: 2^12 points
    constexpr int R0 = 1 << plan_lr(LG, 0), S0 = m / R0;
    constexpr int RH = 1 << plan_lr(LGH, 0), SH = MH / RH, NPH = plan_P(LGH);
    static_assert(M == m && S0 == T && SH <= T, "one first-pass group per thread");
    extern __shared__ float2 sm[];
    const PairSmem s = pair_carve<LG>(sm);
    cg::cluster_group cluster = cg::this_cluster();
    const int cr = (int)cluster.block_rank();
    float2 *recv = reinterpret_cast<float2 *>(s.stage);            // [MH]: the partner's z
    float2 *twh = recv + MH;                                       // middle-pass twiddles of the half-length inverse
    float2 *precv = cluster.map_shared_rank(recv, cr ^ 1);
    pair_tables<LG>(s);
    build_middle_tables<LGH>(twh, threadIdx.x, T);
    const int j = threadIdx.x;
    const float2 tcj = unit_root(j, 2 * L);   // W_N^j
    cluster.sync();   // both CTAs run before either reaches into the other's memory
    float2 *X = s.b0;   // the length-MH inverse transform of this CTA's parity
    bool first = true;
    for (int h = blockIdx.x / 2; h < H; h += gridDim.x / 2) {
        float *Kh = K + (size_t)h * L;
        // ---- Z[2k' + cr] at the digit-reversed position of k' (k and M - k from one pair of loads)
        for (int i = j; i <= MH / 2; i += T) {
            const int k = 2 * i + cr;
            if (k > M / 2) break;
            float2 A, Bc;
            if (k == 0) {
                A = make_float2(__ldcg(Kh), 0.0f);
                Bc = make_float2(__ldcg(Kh + 1), 0.0f);
            } else {
                A = __ldcg(reinterpret_cast<const float2 *>(Kh) + k);
                Bc = cconj(__ldcg(reinterpret_cast<const float2 *>(Kh) + (M - k)));
            }
            float sn, cs;
            sincospif(2.0f * (float)k / (float)L, &sn, &cs);   // w^k = cs + i sn
            const float2 wk = make_float2(cs, sn);
            X[pidx(digrev_inv<LGH>(k >> 1))] = cadd(cadd(A, Bc), mul_i<+1>(cmul(wk, csub(A, Bc))));
            if (k != 0 && k != M / 2) {   // Z[M - k]: A' = conj Bc, Bc' = conj A, w^{M-k} = -conj w^k
                const float2 A2 = cconj(Bc), B2 = cconj(A);
                X[pidx(digrev_inv<LGH>((M - k) >> 1))] =
                    csub(cadd(A2, B2), mul_i<+1>(cmul(cconj(wk), csub(A2, B2))));
            }
        }
        __syncthreads();
        // ---- half-length inverse transform, passes P-1 .. 1, then the last pass in registers
        dit_pass<LGH, NPH - 1, +1, T>(X, twh);
        __syncthreads();
        inverse_middle<LGH, T>(X, twh);
        if (!first) cluster_wait();   // the partner has read the previous channel's hand-over
        if (j < SH) {
            const int o = pidx(j);
            const float2 b = unit_root(j, MH);
            float2 z[RH];
            float2 w = b;
            z[0] = X[o];
            static_for<1, RH>([&](auto q) {
                z[q] = cmulc(X[o + poff<decltype(q)::value * SH>()], w);
                w = cmul(w, b);
            });
            dft<RH, +1>(z);   // z[p] = z_cr[j + p SH]
            static_for<0, RH>([&](auto p) {
                X[o + poff<decltype(p)::value * SH>()] = z[p];   // natural order, own group positions
                precv[j + p * SH] = z[p];
            });
        }
        cluster_arrive_release();
        cluster_wait();   // both halves are in place; both CTAs are done reading the half spectrum
        // ---- chunks x0[k] = K[k], x1[k] = K[k + m] at k = j + p S0
        float2 v0[R0], v1[R0];
        static_for<0, R0>([&](auto p) {
            const int k = j + p * S0, n = k >> 1;
            const float2 zo = X[pidx(n)], zr = recv[n];
            const float2 z0 = cr == 0 ? zo : zr, z1 = cr == 0 ? zr : zo;
            float sn, cs;
            sincospif(2.0f * (float)n / (float)M, &sn, &cs);
            const float2 wz = cmul(make_float2(cs, sn), z1);
            const float2 za = cadd(z0, wz), zb = csub(z0, wz);
            const float ka = (k & 1) ? za.y : za.x, kb = (k & 1) ? zb.y : zb.x;
            Kh[k + cr * m] = cr == 0 ? ka : kb;
            quad_inputs<decltype(p)::value>(cr, make_float2(ka, 0.0f), make_float2(kb, 0.0f), v0[p], v1[p]);
        });
        __syncthreads();   // X (in b0) is read: the first pass may overwrite it
        if (cr == 0) first_pass_halves2<LG, false>(s, v0, v1, j, make_float2(1.0f, 0.0f));
        else first_pass_halves2<LG, true>(s, v0, v1, j, tcj);
        cluster_arrive_relaxed();   // the values read from recv went into the stores above
        first = false;
        __syncthreads();
        float4 *sh = reinterpret_cast<float4 *>(spec + (size_t)h * 2 * L);
        spectrum_tail2<LG>(s, D != nullptr ? __ldg(D + h) : 0.0f, 1.0f / (float)(2 * L), sh + (size_t)cr * (m / 2),
                           sh + (size_t)(cr + 2) * (m / 2));
        __syncthreads();
    }
    if (!first) cluster_wait();   // pairs the last arrive
}

// =============================================================== host side ==
namespace {
LaunchInfo g_quad_conv[2], g_quad_kspec[2];

// Ki non-null: the spectrum of K + i Ki
cudaError_t quad_kspec(const float *K, const float *D, int H, void *ws, cudaStream_t st, const float *Ki) {
    constexpr size_t smem = pair_smem_bytes<kQuadLG>(0);
    const bool cplx = Ki != nullptr;
    auto kern = cplx ? k_kspec_quad<true> : k_kspec_quad<false>;
    int res = 0;
    cudaError_t e = resident_units(kern, g_quad_kspec[cplx], 1, pair_threads<kQuadLG>(), smem, &res);
    if (e != cudaSuccess) return e;
    kern<<<res < 2 * H ? res : 2 * H, pair_threads<kQuadLG>(), smem, st>>>(K, Ki, D, H, (float2 *)ws);
    return cudaGetLastError();
}

LaunchInfo g_quad_half;

// K holds the packed half spectrum on entry and the kernel on exit
cudaError_t quad_kspec_half(float *K, const float *D, int H, void *ws, cudaStream_t st) {
    constexpr size_t smem = pair_smem_bytes<kQuadLG>(0);
    constexpr int T = pair_threads<kQuadLG>();
    int res = 0;
    cudaError_t e = resident_units(k_kspec_quad_half, g_quad_half, 2, T, smem, &res);
    if (e != cudaSuccess) return e;
    const int ncl = res < H ? res : H;
    e = launch_clustered(k_kspec_quad_half, 2, ncl, T, smem, st, K, D, H, (float2 *)ws);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

cudaError_t quad_conv(const float *u, const void *ws, int Bt, int H, float *y, bool adjoint, cudaStream_t st) {
    constexpr size_t smem = pair_smem_bytes<kQuadLG>(0);
    constexpr int T = pair_threads<kQuadLG>();
    auto kern = adjoint ? k_fftconv_quad<true> : k_fftconv_quad<false>;
    int res = 0;
    cudaError_t e = resident_units(kern, g_quad_conv[adjoint], 2, T, smem, &res);
    if (e != cudaSuccess) return e;
    const long long npairs = (long long)H * ((Bt + 1) / 2);
    const int ncl = (long long)res < npairs ? res : (int)npairs;
    e = launch_clustered(kern, 2, ncl, T, smem, st, u, (const float2 *)ws, Bt, H, y);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}
}  // namespace

cudaError_t launch_kspec_l16k(const float *K, const float *D, int H, void *ws, cudaStream_t st, const float *Ki) {
    return quad_kspec(K, D, H, ws, st, Ki);
}
cudaError_t launch_fftconv_l16k(const float *u, const void *ws, int Bt, int H, float *y, bool adjoint,
                                cudaStream_t st) {
    return quad_conv(u, ws, Bt, H, y, adjoint, st);
}
cudaError_t launch_kspec_from_half_l16k(float *K, const float *D, int H, void *ws, cudaStream_t st) {
    return quad_kspec_half(K, D, H, ws, st);
}

}  // namespace s4
