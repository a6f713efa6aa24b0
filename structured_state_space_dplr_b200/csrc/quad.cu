// quad.cu -- the convolution at L = 16384 ("The S4 kernel, from scratch", §5
// fft_conv): the zero-padded length-2L transform split four ways over a
// cluster of two CTAs, each holding two ranks as the two halves of the
// one-CTA pair kernel (pairs.cuh); the split is described in quad.cuh.
//
// k_fftconv_quad : the convolution, persistent over row pairs (CONJ: the
//                  adjoint, with the conjugate spectrum).
#include "quad.cuh"

namespace cg = cooperative_groups;

namespace s4 {

// a hint that brings the line holding p into L2 (no registers, no completion)
__device__ __forceinline__ void l2_prefetch(const void *p) {
    asm volatile("prefetch.global.L2 [%0];" ::"l"(__cvta_generic_to_global(p)));
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
        // the middle passes with warp-level barriers (warp_local_middle, fft.cuh)
        static_assert(warp_local_middle<LG, T, 2>(), "the 16 x 32 x 16 plan on 512 threads");
        const float2 *sh = spec + (size_t)r.h * 2 * L;
        pass_x2<LG, 1, -1, false, T>(s.b0, s.b1, s.tws);
        __syncwarp();
        fused_blocks<LG, 2, CONJ>(s.b0, s.b1, reinterpret_cast<const float4 *>(sh + (size_t)cr * m),
                                  reinterpret_cast<const float4 *>(sh + (size_t)(cr + 2) * m));
        __syncwarp();
        pass_x2<LG, 1, +1, true, T>(s.b0, s.b1, s.tws);
        __syncthreads();
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

namespace {
LaunchInfo g_quad_conv[2];

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

cudaError_t launch_fftconv_l16k(const float *u, const void *ws, int Bt, int H, float *y, bool adjoint,
                                cudaStream_t st) {
    return quad_conv(u, ws, Bt, H, y, adjoint, st);
}

}  // namespace s4
