// spectral.cu -- zero-padded causal FFT convolution and the inverse real FFT
// that turns the DPLR spectrum into the kernel K.
//
// Convolution ("The S4 kernel, from scratch", §5 fft_conv; D u from §1):
//   y[b,h,t] = sum_{s<=t} K[h,s] u[b,h,t-s] + D[h] u[b,h,t],
// computed with length N = 2L transforms so the circular product has no
// wrap-around. Two rows (b, b+1) of one channel are packed as u_b + i u_{b+1}
// (K is real, so the product keeps the rows apart: real part -> row b,
// imaginary part -> row b+1). Up to L = 8192 one CTA holds a row pair's
// whole transform as two halves (pairs.cuh); L = 16384 is a cluster of two
// (quad.cu); longer transforms are split over a cluster of C CTAs (see
// fft.cuh), and because only the first L inputs are nonzero only C/2 input
// chunks enter, and because only the first L outputs are kept the cluster
// combine produces only C/2 of its C output chunks.
//
// k_kspec      : spectrum of the zero-padded K, once per call, shared by all
//                rows; stored per (h, rank) in the digit-reversed order the
//                convolution produces, scaled by 1/N.
// k_fftconv    : persistent clusters; each cluster loops over row pairs:
//                forward transform, product, inverse transform, combine over
//                distributed shared memory, + D u, store.
// k_irfft      : K[h, 0..L) from the packed half spectrum (two channels per
//                complex transform), in place.
#include <atomic>
#include <cooperative_groups.h>

#include "cluster.cuh"
#include "fft.cuh"
#include "launch.h"
#include "pairs.cuh"

namespace cg = cooperative_groups;

namespace s4 {

template <int LG>
__host__ __device__ constexpr int threads_for() {
    return (1 << LG) / 16 < 32 ? 32 : ((1 << LG) / 16 > 512 ? 512 : (1 << LG) / 16);
}
// threads and CTAs per SM of the C-way cluster kernels: a split 16 ways keeps
// two 256-thread CTAs on an SM (registers and shared memory for both)
template <int LG, int C>
__host__ __device__ constexpr int cl_threads() { return C >= 16 ? 256 : threads_for<LG>(); }
template <int C>
__host__ __device__ constexpr int cl_min_blocks() { return C >= 16 ? 2 : 1; }

// dynamic shared memory of the C-way split kernels, in float2:
// buf | tws | ta[S0] | tb[S0] | pre[32] | wcr[8]
template <int LG>
__host__ __device__ constexpr int smem_f2() {
    return (padded(1 << LG) + plan_tw_size(LG) + 2 * ((1 << LG) >> plan_lr(LG, 0)) + 32 + 8 + 1) / 2 * 2;
}

struct Smem {
    float2 *buf, *tws, *ta, *tb, *pre, *wcr;
};
template <int LG>
__device__ __forceinline__ Smem carve(float2 *sm) {
    constexpr int S0 = (1 << LG) >> plan_lr(LG, 0);
    Smem s;
    s.buf = sm;
    s.tws = sm + padded(1 << LG);
    s.ta = s.tws + plan_tw_size(LG);
    s.tb = s.ta + S0;
    s.pre = s.tb + S0;
    s.wcr = s.pre + 32;
    return s;
}

// ------------------------------------------------------------------ kspec --
// spec[h][c][pos] = (FFT_2L(K_h zero-padded)[f] + D_h) / 2L for the frequency
// f = C f' + c held at pos: the spectrum of K + D delta_0, so the convolution
// adds the D u term with no extra pass over u. CPLX: the input is the
// complex signal K + i Ki (Ki [H, L]); its spectrum then has no conjugate
// symmetry, which the convolution does not assume.
// The same spectrum for the cluster convolution (L >= 32768), one cluster of
// C CTAs per channel (persistent over channels), CTA c producing rank c.
// Rank c's input v_c[k] = W_N^{kc} sum_{q < C/2} W_C^{qc} K[k + q m] is formed
// cooperatively as in k_fftconv: CTA c reads K (and Ki) once for its slice of
// positions, runs the length-C DFT of the chunks and stores each rank's value
// into that rank's buffer (distributed shared memory). Barriers: release /
// acquire around those stores; a relaxed arrive after the rank's spectrum is
// stored (its buffer is no longer read), waited on before the next channel's
// stores.
template <int LG, int C, bool CPLX>
__global__ void __launch_bounds__(cl_threads<LG, C>(), cl_min_blocks<C>())
k_kspec_cl(const float *__restrict__ K, const float *__restrict__ Ki, const float *__restrict__ D, int H, int L,
           float2 *__restrict__ spec) {
    constexpr int m = 1 << LG, T = cl_threads<LG, C>();
    constexpr int SL = m / C, S0 = m >> plan_lr(LG, 0);
    extern __shared__ float2 sm[];
    const Smem s = carve<LG>(sm);
    cg::cluster_group cluster = cg::this_cluster();
    const int c = (int)cluster.block_rank();
    const int cl = blockIdx.x / C, ncl = gridDim.x / C;
    float2 *rbuf[C];
    static_for<0, C>([&](auto cc) { rbuf[cc] = cluster.map_shared_rank(s.buf, (int)cc); });
    build_rank_tables<LG>(s.ta, s.tb, s.pre, C, c, threadIdx.x, T);
    build_middle_tables<LG>(s.tws, threadIdx.x, T);
    cluster.sync();   // every CTA of the cluster runs before any reaches into its memory
    const float scale = 1.0f / (float)(C * m);
    bool first = true;
    for (int h = cl; h < H; h += ncl) {
        const float *Kh = K + (size_t)h * L;
        const float *Kih = CPLX ? Ki + (size_t)h * L : nullptr;
        const float Dh = D != nullptr ? __ldg(D + h) : 0.0f;
        if (!first) cluster_wait();   // every rank's buffer is free (previous channel done)
        first = false;
        for (int i = threadIdx.x; i < SL; i += T) {
            const int k = c * SL + i;
            float2 x[C];
            static_for<0, C / 2>([&](auto q) {
                x[q] = make_float2(__ldg(Kh + k + q * m), CPLX ? __ldg(Kih + k + q * m) : 0.0f);
            });
            static_for<C / 2, C>([&](auto q) { x[q] = make_float2(0.0f, 0.0f); });
            dft<C, -1>(x);
            static_for<0, C>([&](auto r) { rbuf[r][pidx(k)] = x[r]; });
        }
        cluster_arrive_release();
        cluster_wait();
        for (int j = threadIdx.x; j < S0; j += T) {
            float2 x[1 << plan_lr(LG, 0)];
            first_group_rec<LG>(x, j, s.ta, s.tb, s.pre, [&](int k) { return s.buf[pidx(k)]; });
            store_first_group<LG>(s.buf, x, j);
        }
        __syncthreads();
        forward_middle<LG, T>(s.buf, s.tws);
        float4 *out = reinterpret_cast<float4 *>(spec + ((size_t)h * C + c) * m);
        forward_last<LG, T>(s.buf, [&](int base, auto &x) {
            constexpr int R = sizeof(x) / sizeof(float2);
            static_for<0, R / 2>([&](auto i) {
                out[spec4_index<LG>(base, i)] = make_float4((x[2 * i].x + Dh) * scale, x[2 * i].y * scale,
                                                (x[2 * i + 1].x + Dh) * scale, x[2 * i + 1].y * scale);
            });
        });
        // the buffer was read into the stores above: partners may write it again
        cluster_arrive_relaxed();
    }
    if (!first) cluster_wait();   // pairs the last arrive
}

// ---------------------------------------------------------------- fftconv --
// L >= 32768: a cluster of C CTAs per row pair, CTA c holding rank c (the
// frequencies C f + c, m = 2L / C points), persistent over row pairs. Rank c's
// input is v_c[k] = W_N^{kc} sum_{q < C/2} W_C^{qc} x_q[k] from the C/2
// nonzero input chunks x_q[k] = (u0 + i u1)[k + q m]. The C CTAs form these
// cooperatively: CTA c takes the positions k of its slice [c m/C, (c+1) m/C),
// loads the chunks of both rows once, runs the length-C DFT of
// [x_0 .. x_{C/2-1}, 0 ..] and stores each rank r's value straight into CTA
// r's buffer at k (distributed shared memory). After a cluster barrier every
// CTA runs its first pass in place (the twist W_N^{kc} from its rank tables),
// the transform, the product with its spectrum rank, the inverse; the C
// partial results are then combined over distributed shared memory, rank c
// writing the outputs t' = c SL + i + r m (r < C/2) of its slice:
//   x[t' + r m] = sum_c W_C^{-c r} (W_N^{-c t'} Z_c[t']).
// Barriers: the buffers are overwritten by the next pair's stores only after
// every CTA's relaxed arrive that follows its combine's output stores (which
// consume every remote value read).
template <int LG, int C, bool CONJ>
__global__ void __launch_bounds__(cl_threads<LG, C>(), cl_min_blocks<C>())
k_fftconv(const float *__restrict__ u, const float2 *__restrict__ spec, int Bt, int H, int L, float *__restrict__ y) {
    constexpr int m = 1 << LG, T = cl_threads<LG, C>();
    constexpr int SL = m / C;                     // slice of positions per rank
    constexpr int R0 = 1 << plan_lr(LG, 0), S0 = m / R0;
    static_assert(C >= 2, "the convolution uses at least two ranks");
    extern __shared__ float2 sm[];
    const Smem s = carve<LG>(sm);
    cg::cluster_group cluster = cg::this_cluster();
    const int c = (int)cluster.block_rank();
    const int cl = blockIdx.x / C, ncl = gridDim.x / C;
    float2 *rbuf[C];
    static_for<0, C>([&](auto cc) { rbuf[cc] = cluster.map_shared_rank(s.buf, (int)cc); });
    build_rank_tables<LG>(s.ta, s.tb, s.pre, C, c, threadIdx.x, T);
    build_middle_tables<LG>(s.tws, threadIdx.x, T);
    cluster.sync();   // every CTA of the cluster runs before any reaches into its memory

    const int nbp = (Bt + 1) / 2;
    const long long npairs = (long long)H * nbp;
    bool first = true;
    for (long long pr = cl; pr < npairs; pr += ncl) {
        const int h = (int)(pr / nbp), b0 = 2 * (int)(pr % nbp);
        const bool has1 = (b0 + 1) < Bt;
        const float *u0 = u + ((size_t)b0 * H + h) * L;
        const float *u1 = has1 ? u0 + (size_t)H * L : u0;
        // ---- every rank's first-pass input, from this CTA's slice of positions
        if (!first) cluster_wait();   // all buffers are read (previous combine)
        first = false;
        for (int i = threadIdx.x; i < SL; i += T) {
            const int k = c * SL + i;
            float2 x[C];
            static_for<0, C / 2>([&](auto q) {
                x[q] = make_float2(__ldg(u0 + k + q * m), has1 ? __ldg(u1 + k + q * m) : 0.0f);
            });
            static_for<C / 2, C>([&](auto q) { x[q] = make_float2(0.0f, 0.0f); });
            dft<C, -1>(x);   // x[r] = sum_q W_C^{q r} x_q
            static_for<0, C>([&](auto r) { rbuf[r][pidx(k)] = x[r]; });
        }
        cluster_arrive_release();
        cluster_wait();
        // ---- first pass in place, then the transform
        for (int j = threadIdx.x; j < S0; j += T) {
            float2 x[R0];
            first_group_rec<LG>(x, j, s.ta, s.tb, s.pre, [&](int k) { return s.buf[pidx(k)]; });
            store_first_group<LG>(s.buf, x, j);
        }
        __syncthreads();
        const float4 *sp = reinterpret_cast<const float4 *>(spec + ((size_t)h * C + c) * m);
        if constexpr (warp_local_middle<LG, T, 1>()) {   // barriers between the middle passes per warp
            dif_pass<LG, 1, -1, T>(s.buf, s.tws);
            __syncwarp();
            fused_blocks<LG, 1, CONJ>(s.buf, nullptr, sp, nullptr);
            __syncwarp();
            dit_pass<LG, 1, +1, T>(s.buf, s.tws);
            __syncthreads();
        } else {
        forward_middle<LG, T>(s.buf, s.tws);
        fused_middle<LG, T>(s.buf, [&](int base, auto &x) {
            constexpr int R = sizeof(x) / sizeof(float2);
            static_for<0, R / 2>([&](auto i) {
                const float4 k2 = __ldg(sp + spec4_index<LG>(base, i));
                if constexpr (CONJ) {
                    x[2 * i] = cmulc(x[2 * i], make_float2(k2.x, k2.y));
                    x[2 * i + 1] = cmulc(x[2 * i + 1], make_float2(k2.z, k2.w));
                } else {
                    x[2 * i] = cmul(x[2 * i], make_float2(k2.x, k2.y));
                    x[2 * i + 1] = cmul(x[2 * i + 1], make_float2(k2.z, k2.w));
                }
            });
        });
        __syncthreads();
        inverse_middle<LG, T>(s.buf, s.tws);
        }
        inverse_last_rec<LG, T>(s.buf, s.ta, s.tb, s.pre);
        cluster_arrive_release();
        cluster_wait();
        // ---- combine the C partial transforms; rank c writes t' in [c SL, (c+1) SL)
        float *y0 = y + ((size_t)b0 * H + h) * L;
        float *y1 = y0 + (size_t)H * L;
        constexpr int PER = SL / T > 0 ? (SL / T < 4 ? SL / T : 4) : 1;   // elements per batch
        for (int i0 = threadIdx.x; i0 < SL; i0 += T * PER) {
            float2 w[PER][C];
            static_for<0, PER>([&](auto e) {
                const int i = i0 + e * T;
                static_for<0, C>([&](auto cc) {
                    w[e][cc] = (i < SL) ? rbuf[cc][pidx(c * SL + i)] : make_float2(0.f, 0.f);
                });
            });
            static_for<0, PER>([&](auto e) {
                const int i = i0 + e * T;
                if (i < SL) {
                    static_for<0, C / 2>([&](auto r) {
                        float2 o = w[e][0];
                        static_for<1, C>([&](auto cc) {
                            o = cadd(o, rot<decltype(cc)::value * decltype(r)::value, C, +1>(w[e][cc]));
                        });
                        const int t = c * SL + i + r * m;
                        y0[t] = o.x;
                        if (has1) y1[t] = o.y;
                    });
                }
            });
        }
        cluster_arrive_relaxed();   // after the stores that consume every remote value read
    }
    // the partners may still read this CTA's buffer: wait before exiting
    if (!first) cluster_wait();
}

// ------------------------------------------------------- fftconv, one CTA --
// L <= 8192: one CTA per row pair holds both halves of the length-2L
// transform; see conv_pair (pairs.cuh). Persistent: the next row pair is
// staged with cp.async while the current one is transformed.
template <int LG, bool CONJ>
__global__ void __launch_bounds__(pair_threads<LG>(), pair_min_blocks<LG>())
k_fftconv_pair(const float *__restrict__ u, const float2 *__restrict__ spec, int Bt, int H, int L,
               float *__restrict__ y) {
    extern __shared__ float2 sm[];
    const PairSmem s = pair_carve<LG>(sm);
    pair_tables<LG>(s);
    const long long npairs = (long long)H * ((Bt + 1) / 2);
    if ((long long)blockIdx.x < npairs) pair_stage_rows<LG>(s, u, Bt, H, blockIdx.x);
    for (long long pr = blockIdx.x; pr < npairs; pr += gridDim.x) {
        const RowPair r = row_pair(pr, Bt);
        cp_async_wait_all();
        __syncthreads();   // stage ready; previous pair's buffers no longer read
        float *y0 = y + ((size_t)r.b0 * H + r.h) * L;
        conv_pair<LG, CONJ>(s, spec + (size_t)r.h * 2 * L, y0, y0 + (size_t)H * L, r.has1, [&] {
            if (pr + gridDim.x < npairs) pair_stage_rows<LG>(s, u, Bt, H, pr + gridDim.x);
        });
    }
}

// The spectrum k_fftconv_pair reads, from K in global memory: one CTA per
// channel, both halves of the length-2L transform (see kspec_channel).
template <int LG>
__global__ void __launch_bounds__(pair_threads<LG>(), pair_min_blocks<LG>())
k_kspec_pair(const float *__restrict__ K, const float *__restrict__ D, int H, float2 *__restrict__ spec) {
    extern __shared__ float2 sm[];
    const PairSmem s = pair_carve<LG>(sm);
    pair_tables<LG>(s);
    __syncthreads();
    for (int h = blockIdx.x; h < H; h += gridDim.x) {
        kspec_channel<LG>(s, K + (size_t)h * (1 << LG), D != nullptr ? __ldg(D + h) : 0.0f,
                          spec + (size_t)h * 2 * (1 << LG));
        __syncthreads();   // the buffers are reused by the next channel
    }
}

// ------------------------------------------------------------------ irfft --
__device__ __forceinline__ float2 half_spec(const float *Kh, int f, int L) {
    if (f == 0) return make_float2(Kh[0], 0.0f);
    if (f == L / 2) return make_float2(Kh[1], 0.0f);
    if (f < L / 2) return reinterpret_cast<const float2 *>(Kh)[f];
    return cconj(reinterpret_cast<const float2 *>(Kh)[L - f]);
}

// Split 8 ways or more, two 256-thread CTAs share an SM, so twice the
// clusters are resident: at L = 65536 (H = 64) all 32 channel pairs run at
// once on 37 clusters of 8 instead of two rounds on 18, 65 -> 47 us.
template <int LG, int C>
__host__ __device__ constexpr int irfft_threads() { return C >= 8 ? 256 : threads_for<LG>(); }
template <int C>
__host__ __device__ constexpr int irfft_min_blocks() { return C >= 8 ? 2 : 1; }
template <int LG, int C>
__global__ void __launch_bounds__(irfft_threads<LG, C>(), irfft_min_blocks<C>())
k_irfft(float *K, int H, int L) {
    constexpr int m = 1 << LG, T = irfft_threads<LG, C>(), P = plan_P(LG);
    constexpr int SL = m / C;
    extern __shared__ float2 sm[];
    const Smem s = carve<LG>(sm);
    int c = 0, cl = blockIdx.x, ncl = gridDim.x;
    if constexpr (C > 1) {
        c = (int)cg::this_cluster().block_rank();
        cl = blockIdx.x / C;
        ncl = gridDim.x / C;
    }
    build_rank_tables<LG>(s.ta, s.tb, s.pre, C, c, threadIdx.x, T);
    build_middle_tables<LG>(s.tws, threadIdx.x, T);
    if constexpr (C > 1) cg::this_cluster().sync(); else __syncthreads();
    const int npairs = (H + 1) / 2;
    for (int pr = cl; pr < npairs; pr += ncl) {
        float *K1 = K + (size_t)(2 * pr) * L;
        const bool has2 = 2 * pr + 1 < H;
        float *K2 = has2 ? K1 + L : K1;
        auto value = [&](int f) {   // the two channels' half spectra packed as a + i b
            const float2 a = half_spec(K1, f, L);
            const float2 b = has2 ? half_spec(K2, f, L) : make_float2(0.0f, 0.0f);
            return make_float2(a.x - b.y, a.y + b.x);
        };
        if constexpr (C >= 4) {
            // cooperative gather: this CTA reads the frequencies of its
            // contiguous slice (coalesced) and stores each one at its digit-
            // reversed position in the buffer of the rank f mod C that owns it
            // (a strided gather of every C-th frequency fetches each 32-byte
            // sector once per CTA: 56.0 against 66.5 us at C = 8; at C = 2
            // the strided form is the faster, 29.6 against 35.5 us)
            // Loads go out NB at a time before their stores (one L2 latency per
            // batch), without branches: f < L/2 reads X[f] (f = 0: the word
            // (K[0], K[1]) holding X_0 and X_{L/2}), f > L/2 conj X[L - f],
            // f = L/2 that first word again.
            cg::cluster_group cluster = cg::this_cluster();
            constexpr int NB = 8;
            static_assert(m % (T * NB) == 0, "whole batches");
            const float2 *X1 = reinterpret_cast<const float2 *>(K1);
            const float2 *X2 = reinterpret_cast<const float2 *>(K2);
            for (int i0 = threadIdx.x; i0 < m; i0 += T * NB) {
                float2 va[NB], vb[NB];
                static_for<0, NB>([&](auto e) {
                    const int f = c * m + i0 + decltype(e)::value * T;
                    const int w = f < L / 2 ? f : (f == L / 2 ? 0 : L - f);
                    va[e] = __ldcg(X1 + w);
                    vb[e] = has2 ? __ldcg(X2 + w) : make_float2(0.0f, 0.0f);
                });
                static_for<0, NB>([&](auto e) {
                    const int f = c * m + i0 + decltype(e)::value * T;
                    float2 a = va[e], b = vb[e];
                    if (f == 0) {
                        a.y = 0.0f;
                        b.y = 0.0f;
                    } else if (f == L / 2) {
                        a = make_float2(a.y, 0.0f);
                        b = make_float2(b.y, 0.0f);
                    } else if (f > L / 2) {
                        a = cconj(a);
                        b = cconj(b);
                    }
                    const int r = f % C, fr = f / C;
                    cluster.map_shared_rank(s.buf, r)[pidx(digrev_inv<LG>(fr))] =
                        make_float2(a.x - b.y, a.y + b.x);
                });
            }
            cluster.sync();
        } else {
            gather_digit_reversed<LG, T>(s.buf, [&](int fr) { return value(C * fr + c); });
            __syncthreads();
        }
        dit_pass<LG, P - 1, +1, T>(s.buf, s.tws);
        __syncthreads();
        inverse_middle<LG, T>(s.buf, s.tws);
        inverse_last_rec<LG, T>(s.buf, s.ta, s.tb, s.pre);
        if constexpr (C > 1) cg::this_cluster().sync(); else __syncthreads();
        for (int i = threadIdx.x; i < SL; i += T) {
            const int tp = c * SL + i;
            float2 w[C];
            if constexpr (C > 1) {
                static_for<0, C>([&](auto cc) { w[cc] = cg::this_cluster().map_shared_rank(s.buf, (int)cc)[pidx(tp)]; });
            } else {
                w[0] = s.buf[pidx(tp)];
            }
            static_for<0, C>([&](auto r) {
                float2 o = w[0];
                static_for<1, C>([&](auto cc) {
                    o = cadd(o, rot<decltype(cc)::value * decltype(r)::value, C, +1>(w[cc]));
                });
                K1[tp + r * m] = o.x;
                if (has2) K2[tp + r * m] = o.y;
            });
        }
        if constexpr (C > 1) cg::this_cluster().sync(); else __syncthreads();
    }
}

// =============================================================== host side ==
namespace {

size_t align256(size_t b) { return (b + 255) & ~size_t(255); }

// ---- convolution / kspec instantiation for one L ----
// C == 2 with LG <= 13: the one-CTA pair kernels (L <= 8192); otherwise the
// C-way cluster kernels (L >= 32768; L = 16384 has its own in quad.cu).
template <int LG, int C>
struct ConvKernels {
    static constexpr int T = cl_threads<LG, C>();
    static constexpr size_t smem = sizeof(float2) * (size_t)smem_f2<LG>();
    static constexpr bool kPair = C == 2 && LG <= 13;
    static LaunchInfo info_conv[2], info_kspec, info_kspec_c, info_kspec_pair, info_pair[2];

    // Ki non-null: the spectrum of K + i Ki (cluster paths only)
    static cudaError_t kspec(const float *K, const float *D, int H, int L, void *ws, cudaStream_t st,
                             const float *Ki = nullptr) {
        float2 *spec = (float2 *)ws;
        if constexpr (kPair) {
            if (Ki != nullptr) return cudaErrorInvalidValue;
            // the one-CTA convolution's spectrum: persistent, one channel per CTA at a time
            auto kern = k_kspec_pair<LG>;
            constexpr size_t psmem = pair_smem_bytes<LG>(0);
            int res = 0;
            cudaError_t e = resident_units(kern, info_kspec_pair, 1, pair_threads<LG>(), psmem, &res);
            if (e != cudaSuccess) return e;
            kern<<<res < H ? res : H, pair_threads<LG>(), psmem, st>>>(K, D, H, spec);
            return cudaGetLastError();
        } else {
            auto kern = Ki != nullptr ? k_kspec_cl<LG, C, true> : k_kspec_cl<LG, C, false>;
            int res = 0;
            cudaError_t e = resident_units(kern, Ki != nullptr ? info_kspec_c : info_kspec, C, T, smem, &res);
            if (e != cudaSuccess) return e;
            const int ncl = res < H ? res : H;
            e = launch_clustered(kern, C, ncl, T, smem, st, K, Ki, D, H, L, spec);
            if (e != cudaSuccess) return e;
            return cudaGetLastError();
        }
    }

    static cudaError_t conv(const float *u, const void *ws, int Bt, int H, int L, float *y, bool adjoint,
                            cudaStream_t st) {
        const float2 *spec = (const float2 *)ws;
        const long long npairs = (long long)H * ((Bt + 1) / 2);
        if constexpr (kPair) {
            // one CTA per row pair, both halves in one CTA; persistent grid
            auto kern = adjoint ? k_fftconv_pair<LG, true> : k_fftconv_pair<LG, false>;
            constexpr int TT = pair_threads<LG>();
            constexpr size_t psmem = pair_smem_bytes<LG>(0);
            int res = 0;
            cudaError_t e = resident_units(kern, info_pair[adjoint], 1, TT, psmem, &res);
            if (e != cudaSuccess) return e;
            const int grid = (long long)res < npairs ? res : (int)npairs;
            kern<<<grid, TT, psmem, st>>>(u, spec, Bt, H, L, y);
            return cudaGetLastError();
        } else {
            auto kern = adjoint ? k_fftconv<LG, C, true> : k_fftconv<LG, C, false>;
            int res = 0;
            cudaError_t e = resident_units(kern, info_conv[adjoint], C, T, smem, &res);
            if (e != cudaSuccess) return e;
            const int ncl = (long long)res < npairs ? res : (int)npairs;
            e = launch_clustered(kern, C, ncl, T, smem, st, u, spec, Bt, H, L, y);
            if (e != cudaSuccess) return e;
            return cudaGetLastError();
        }
    }
};
template <int LG, int C> LaunchInfo ConvKernels<LG, C>::info_conv[2];
template <int LG, int C> LaunchInfo ConvKernels<LG, C>::info_kspec;
template <int LG, int C> LaunchInfo ConvKernels<LG, C>::info_kspec_c;
template <int LG, int C> LaunchInfo ConvKernels<LG, C>::info_kspec_pair;
template <int LG, int C> LaunchInfo ConvKernels<LG, C>::info_pair[2];

// ---- irfft instantiation ----
template <int LG, int C>
struct IrfftKernels {
    static constexpr int T = irfft_threads<LG, C>();
    static constexpr size_t smem = sizeof(float2) * (size_t)smem_f2<LG>();
    static LaunchInfo info;
    static cudaError_t run(float *K, int H, int L, cudaStream_t st) {
        auto kern = k_irfft<LG, C>;
        int res = 0;
        cudaError_t e = resident_units(kern, info, C, T, smem, &res);
        if (e != cudaSuccess) return e;
        const int npairs = (H + 1) / 2;
        int ncl = res < npairs ? res : npairs;
        e = launch_clustered(kern, C, ncl, T, smem, st, K, H, L);
        if (e != cudaSuccess) return e;
        return cudaGetLastError();
    }
};
template <int LG, int C> LaunchInfo IrfftKernels<LG, C>::info;

}  // namespace

// Cluster split of the length-2L convolution transform: C ranks of m = 2L/C
// points (C = 2 up to L = 8192 is the one-CTA pair kernel's two halves). At
// L = 65536 the split is 16 ways (a cluster of 16, beyond the portable size,
// two 256-thread CTAs per SM): 219 us against 231 us for 8 ranks of 2^14
// points at H = 64, batch 4, where one 156 KB CTA per SM left 28 SMs idle
// (15 clusters of 8 fit).
ConvGeom conv_geom(int L) {
    switch (L) {
        case 16: return {2, 4};
        case 32: return {2, 5};
        case 64: return {2, 6};
        case 128: return {2, 7};
        case 256: return {2, 8};
        case 512: return {2, 9};
        case 1024: return {2, 10};
        case 2048: return {2, 11};
        case 4096: return {2, 12};
        case 8192: return {2, 13};
        case 16384: return {4, 13};
        case 32768: return {8, 13};
        case 65536: return {16, 13};
        default: return {0, 0};
    }
}

// the workspace holds only the spectrum of K + D delta_0: H x 2L complex values
size_t conv_workspace_bytes(int H, int L) { return align256((size_t)H * 2 * L * sizeof(float2)); }

// (L, log2 m, C)
#define S4_CONV_CASES(X) \
    X(16, 4, 2)          \
    X(32, 5, 2)          \
    X(64, 6, 2)          \
    X(128, 7, 2)         \
    X(256, 8, 2)         \
    X(512, 9, 2)         \
    X(1024, 10, 2)       \
    X(2048, 11, 2)       \
    X(4096, 12, 2)       \
    X(8192, 13, 2)       \
    X(32768, 13, 8)      \
    X(65536, 13, 16)


cudaError_t launch_kspec(const float *K, const float *D, int H, int L, void *ws, cudaStream_t st, const float *Ki) {
    if (L == 16384) return launch_kspec_l16k(K, D, H, ws, st, Ki);
    switch (L) {
#define X(LL, LG, C) case LL: return ConvKernels<LG, C>::kspec(K, D, H, L, ws, st, Ki);
        S4_CONV_CASES(X)
#undef X
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_fftconv(const float *u, const void *ws, int Bt, int H, int L, float *y, cudaStream_t st,
                           bool adjoint) {
    if (L == 16384) return launch_fftconv_l16k(u, ws, Bt, H, y, adjoint, st);
    switch (L) {
#define X(LL, LG, C) case LL: return ConvKernels<LG, C>::conv(u, ws, Bt, H, L, y, adjoint, st);
        S4_CONV_CASES(X)
#undef X
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_kspec_from_half(float *K, const float *D, int H, int L, void *ws, cudaStream_t st) {
    if (L == 16384) return launch_kspec_from_half_l16k(K, D, H, ws, st);
    cudaError_t e = launch_irfft_packed(K, H, L, st);
    if (e == cudaSuccess) e = launch_kspec(K, D, H, L, ws, st);
    return e;
}

cudaError_t launch_irfft_packed(float *K, int H, int L, cudaStream_t st) {
    switch (L) {
        case 16: return IrfftKernels<4, 1>::run(K, H, L, st);
        case 32: return IrfftKernels<5, 1>::run(K, H, L, st);
        case 64: return IrfftKernels<6, 1>::run(K, H, L, st);
        case 128: return IrfftKernels<7, 1>::run(K, H, L, st);
        case 256: return IrfftKernels<8, 1>::run(K, H, L, st);
        case 512: return IrfftKernels<9, 1>::run(K, H, L, st);
        case 1024: return IrfftKernels<10, 1>::run(K, H, L, st);
        case 2048: return IrfftKernels<11, 1>::run(K, H, L, st);
        case 4096: return IrfftKernels<12, 1>::run(K, H, L, st);
        case 8192: return IrfftKernels<13, 1>::run(K, H, L, st);
        case 16384: return IrfftKernels<13, 2>::run(K, H, L, st);
        case 32768: return IrfftKernels<13, 4>::run(K, H, L, st);
        case 65536: return IrfftKernels<13, 8>::run(K, H, L, st);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace s4
