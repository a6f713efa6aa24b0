// quad_spec.cu -- the spectra the L = 16384 convolution reads ("The S4
// kernel, from scratch", §4 kernel via the generating function and its
// inverse FFT, §5 fft_conv), in the four-rank layout of quad.cuh.
//
// k_kspec_quad      : the spectrum of K + D delta_0 from K (or K + i Ki);
// k_kspec_quad_pair : the same for two channels at once from k_cauchy's
//                     packed half spectra, with the inverse real transform
//                     folded in (K stored in place).
#include "quad.cuh"

namespace cg = cooperative_groups;

namespace s4 {

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
// round-trip through memory between the two, for two channels a, b at once:
// one cluster of two CTAs per channel pair. The two half spectra are
// inverted together as Y = X_a + i X_b (a
// length-L complex transform whose output is y = K_a + i K_b), split across
// the CTAs by the parity of the frequency: CTA cr inverts Y[2k' + cr] (m
// points) and, with z_cr its result,
//   y[k] = z_0[k] + W_L^{-k} z_1[k],  y[k + m] = z_0[k] - W_L^{-k} z_1[k]  (k < m).
// The CTAs hand z_cr over with distributed-shared-memory stores into each
// other's stage area (split cluster barrier as in k_fftconv_quad), CTA 0
// stores K[0, m) and CTA 1 K[m, 2m) of both channels in place of the half
// spectra (the exchange's barrier orders those stores after both CTAs' reads
// of them), and y, being K_a + i K_b, enters the forward transform as the
// convolution's row pair u_0 + i u_1 does. The two
// spectra come apart by conjugate symmetry (K_a, K_b real):
//   X_a[f] = (Z[f] + conj Z[N-f]) / 2,  X_b[f] = (Z[f] - conj Z[N-f]) / 2i,
// where N - f of rank c (f = 4f' + c) lies in rank -c mod 4: frequency
// (m - f') mod m of rank 0, else m - 1 - f' of rank 4 - c. Both ranks sit in
// the same CTA (0 and 2 in CTA 0, 1 and 3 in CTA 1), and the position of
// m - 1 - f' is m - 1 - p (the digit reversal permutes bits), so only rank 0
// looks its partners up by frequency.

__global__ void __launch_bounds__(pair_threads<kQuadLG>(), 1)
k_kspec_quad_pair(float *__restrict__ K, const float *__restrict__ D, int H, float2 *__restrict__ spec) {
    constexpr int LG = kQuadLG, m = 1 << LG, L = 2 * m, T = pair_threads<LG>(), P = plan_P(LG);
    constexpr int R0 = 1 << plan_lr(LG, 0), S0 = m / R0;
    constexpr int RL = 1 << plan_lr(LG, P - 1), G = m / RL;
    static_assert(S0 == T, "one first-pass group per thread");
    extern __shared__ float2 sm[];
    const PairSmem s = pair_carve<LG>(sm);
    cg::cluster_group cluster = cg::this_cluster();
    const int cr = (int)cluster.block_rank();
    float2 *recv = reinterpret_cast<float2 *>(s.stage);   // [m]: the partner's z
    float2 *precv = cluster.map_shared_rank(recv, cr ^ 1);
    pair_tables<LG>(s);
    const int j = threadIdx.x;
    const float2 tcj = unit_root(j, 2 * L);   // W_N^j
    const float2 wlj = cconj(unit_root(j, L));   // W_L^{-j}
    cluster.sync();   // both CTAs run before either reaches into the other's memory
    const float scale = 1.0f / (float)(2 * L);
    const int npc = (H + 1) / 2;
    bool first = true;
    for (int pc = blockIdx.x / 2; pc < npc; pc += gridDim.x / 2) {
        const int ha = 2 * pc;
        const bool hasb = ha + 1 < H;
        float *Ka = K + (size_t)ha * L;
        float *Kb = hasb ? Ka + L : Ka;   // channel ha + 1 (read and written only if hasb)
        // ---- Y[2k' + cr] at the digit-reversed position of k', k' = j + q T:
        // all loads first (one L2 latency instead of one per k'), without
        // branches: f < L/2 for q < NQ/2 (X[f]; f = 0 holds X_0 and X_{L/2}
        // as the word (K[0], K[1])), f > L/2 beyond (conj X[L - f]; f = L/2
        // reads that first word too)
        {
            constexpr int NQ = m / T;
            const float2 *Xa = reinterpret_cast<const float2 *>(Ka);
            const float2 *Xb = reinterpret_cast<const float2 *>(Kb);
            float2 va[NQ], vb[NQ];
            static_for<0, NQ>([&](auto qc) {
                constexpr int q = decltype(qc)::value;
                const int f = 2 * (j + q * T) + cr;
                const int w = q < NQ / 2 ? f : (f == L / 2 ? 0 : L - f);
                va[q] = __ldcg(Xa + w);
                vb[q] = hasb ? __ldcg(Xb + w) : make_float2(0.0f, 0.0f);
            });
            static_for<0, NQ>([&](auto qc) {
                constexpr int q = decltype(qc)::value;
                const int kk = j + q * T, f = 2 * kk + cr;
                float2 a = va[q], b = vb[q];
                if constexpr (q < NQ / 2) {
                    if (f == 0) { a.y = 0.0f; b.y = 0.0f; }
                } else if (f == L / 2) {
                    a = make_float2(a.y, 0.0f);
                    b = make_float2(b.y, 0.0f);
                } else {
                    a = cconj(a);
                    b = cconj(b);
                }
                s.b0[pidx(digrev_inv<LG>(kk))] = make_float2(a.x - b.y, a.y + b.x);
            });
        }
        __syncthreads();
        // ---- the length-m inverse: passes P-1 .. 1, then the first pass in registers
        dit_pass<LG, P - 1, +1, T>(s.b0, s.tws);
        __syncthreads();
        inverse_middle<LG, T>(s.b0, s.tws);
        if (!first) cluster_wait();   // the partner has read the previous pair's hand-over
        {
            const int o = pidx(j);
            const float2 bw = s.tb[j];   // W_m^j
            float2 z[R0];
            float2 w = bw;
            z[0] = s.b0[o];
            static_for<1, R0>([&](auto q) {
                z[q] = cmulc(s.b0[o + poff<decltype(q)::value * S0>()], w);
                w = cmul(w, bw);
            });
            dft<R0, +1>(z);   // z[p] = z_cr[j + p S0]
            static_for<0, R0>([&](auto p) {
                s.b0[o + poff<decltype(p)::value * S0>()] = z[p];   // natural order, own group positions
                precv[j + p * S0] = z[p];
            });
        }
        cluster_arrive_release();
        cluster_wait();   // both halves in place; both CTAs are done reading the half spectra
        // ---- y at k = j + p S0 and k + m; this CTA's chunk of K_a, K_b; the forward's inputs
        float2 v0[R0], v1[R0];
        static_for<0, R0>([&](auto pc2) {
            constexpr int p = decltype(pc2)::value;
            const int k = j + p * S0;
            const float2 zo = s.b0[pidx(k)], zr = recv[k];
            const float2 z0 = cr == 0 ? zo : zr, z1 = cr == 0 ? zr : zo;
            const float2 wz = rot<p, 32, +1>(cmul(wlj, z1));   // W_L^{-k} = W_L^{-j} W_32^{-p}
            const float2 ya = cadd(z0, wz), yb = csub(z0, wz);
            const float2 yk = cr == 0 ? ya : yb;
            Ka[k + cr * m] = yk.x;
            if (hasb) Kb[k + cr * m] = yk.y;
            quad_inputs<p>(cr, ya, yb, v0[p], v1[p]);
        });
        __syncthreads();   // b0 is read: the first pass may overwrite it
        if (cr == 0) first_pass_halves2<LG, false>(s, v0, v1, j, make_float2(1.0f, 0.0f));
        else first_pass_halves2<LG, true>(s, v0, v1, j, tcj);
        cluster_arrive_relaxed();   // the values read from recv went into the stores above
        first = false;
        __syncthreads();
        // ---- forward passes 1 .. P-1, the last one back into the buffers
        forward_middle_x2<LG, T>(s.b0, s.b1, s.tws);
        for (int g = j; g < G; g += T) {
            const int o = pidx(g * RL);
            float2 x[RL], z[RL];
            load_contig<RL>(s.b0 + o, x);
            load_contig<RL>(s.b1 + o, z);
            dft<RL, -1>(x);
            dft<RL, -1>(z);
            store_contig<RL>(s.b0 + o, x);
            store_contig<RL>(s.b1 + o, z);
        }
        __syncthreads();
        // ---- the two spectra apart, (X + D) / N, in spec4_index order: each
        // thread takes whole groups of RL positions (16-byte shared-memory
        // loads); the partner group of ranks 1 .. 3 is group G - 1 - g reversed
        const float Da = D != nullptr ? __ldg(D + ha) : 0.0f;
        const float Db = hasb && D != nullptr ? __ldg(D + ha + 1) : 0.0f;
        float4 *sa = reinterpret_cast<float4 *>(spec + (size_t)ha * 2 * L);
        float4 *sb = hasb ? sa + L : sa;   // channel ha + 1: 2L float2 = L float4 on (written only if hasb)
        static_for<0, 2>([&](auto hc) {
            constexpr int half = decltype(hc)::value;   // buffer b0 (rank cr) or b1 (rank cr + 2)
            const float2 *own = half == 0 ? s.b0 : s.b1;
            const float2 *par = (cr == 0) == (half == 0) ? s.b0 : s.b1;   // CTA 0: the same buffer; CTA 1: the other
            const int rank = cr + 2 * half;
            for (int g = j; g < G; g += T) {
                float2 zf[RL], zp[RL];
                load_contig<RL>(own + pidx(g * RL), zf);
                if (rank != 0) {
                    float2 zr[RL];
                    load_contig<RL>(par + pidx((G - 1 - g) * RL), zr);
                    static_for<0, RL>([&](auto r) { zp[r] = zr[RL - 1 - decltype(r)::value]; });
                } else {
                    static_for<0, RL>([&](auto r) {
                        const int q = g * RL + decltype(r)::value;
                        zp[r] = par[pidx(digrev_inv<LG>((m - digrev<LG>(q)) & (m - 1)))];
                    });
                }
                static_for<0, RL / 2>([&](auto ic) {
                    constexpr int i = decltype(ic)::value;
                    const float2 f0 = zf[2 * i], f1 = zf[2 * i + 1], p0 = zp[2 * i], p1 = zp[2 * i + 1];
                    const size_t wi = (size_t)rank * (m / 2) + spec4_index<LG>(g * RL, i);
                    sa[wi] = make_float4((0.5f * (f0.x + p0.x) + Da) * scale, 0.5f * (f0.y - p0.y) * scale,
                                         (0.5f * (f1.x + p1.x) + Da) * scale, 0.5f * (f1.y - p1.y) * scale);
                    if (hasb)
                        sb[wi] = make_float4((0.5f * (f0.y + p0.y) + Db) * scale, 0.5f * (p0.x - f0.x) * scale,
                                             (0.5f * (f1.y + p1.y) + Db) * scale, 0.5f * (p1.x - f1.x) * scale);
                });
            }
        });
        __syncthreads();   // the buffers are gathered into again by the next pair
    }
    if (!first) cluster_wait();   // pairs the last arrive
}

namespace {
LaunchInfo g_quad_kspec[2], g_quad_pair;

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

// K holds the packed half spectra on entry and the kernel on exit
cudaError_t quad_kspec_pair(float *K, const float *D, int H, void *ws, cudaStream_t st) {
    constexpr size_t smem = pair_smem_bytes<kQuadLG>(0);
    constexpr int T = pair_threads<kQuadLG>();
    int res = 0;
    cudaError_t e = resident_units(k_kspec_quad_pair, g_quad_pair, 2, T, smem, &res);
    if (e != cudaSuccess) return e;
    const int npc = (H + 1) / 2;
    const int ncl = res < npc ? res : npc;
    e = launch_clustered(k_kspec_quad_pair, 2, ncl, T, smem, st, K, D, H, (float2 *)ws);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}
}  // namespace

cudaError_t launch_kspec_l16k(const float *K, const float *D, int H, void *ws, cudaStream_t st, const float *Ki) {
    return quad_kspec(K, D, H, ws, st, Ki);
}
cudaError_t launch_kspec_from_half_l16k(float *K, const float *D, int H, void *ws, cudaStream_t st) {
    return quad_kspec_pair(K, D, H, ws, st);
}

}  // namespace s4
