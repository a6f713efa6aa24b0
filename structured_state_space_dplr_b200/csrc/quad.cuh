// quad.cuh -- what the L = 16384 kernels share (quad.cu, quad_spec.cu): the
// split of the zero-padded length-2L transform over a cluster of two CTAs
// ("The S4 kernel, from scratch", §5 fft_conv).
#pragma once
#include <cooperative_groups.h>

#include "cluster.cuh"
#include "fft.cuh"
#include "launch.h"
#include "pairs.cuh"

namespace s4 {

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

}  // namespace s4
