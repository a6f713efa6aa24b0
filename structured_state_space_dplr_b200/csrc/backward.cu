// backward.cu -- gradients of the convolution view ("The S4 kernel, from
// scratch", §5 fft_conv; §6 makes the layer trainable) for L <= 8192:
//
//   du[b,h,s] = sum_{t>=s} K[h,t-s] dy[b,h,t] + D[h] dy[b,h,s]
//             -- the forward convolution kernel with the conjugate spectrum
//                (k_fftconv_pair<LG, true>, spectral.cu);
//   dK[h,k]   = sum_b sum_{t>=k} dy[b,h,t] u[b,h,t-k],   dD[h] = dK[h,0]
//             -- k_corr_pair below.
//
// dK: two rows are packed as for the forward, Zu = FFT_2L(u_b + i u_b+1) and
// Zd = FFT_2L(dy_b + i dy_b+1). With U, D the spectra of the single rows,
//   conj(Zu) Zd = conj(U_b) D_b + conj(U_b+1) D_b+1
//               + i (conj(U_b) D_b+1 - conj(U_b+1) D_b),
// and the inverse transform of each bracket is a real correlation: the two
// wanted correlations land in the real part, the cross terms in the imaginary
// part. So conj(Zu) Zd is summed over the row pairs of a channel (in the
// digit-reversed order the forward passes leave, no reordering) and inverse
// transformed once; the real part of the first L outputs, times 1/2L, is dK.
#include "launch.h"
#include "pairs.cuh"

namespace s4 {

// One CTA per channel at a time (persistent over channels), looping over the
// channel's row pairs. The forward transform of the u pair leaves Zu in the
// channel's scratch slice, that of the dy pair multiplies its last-pass
// groups by conj(Zu) and accumulates into the channel's acc slice; each
// thread owns the same last-pass groups throughout, so the scratch and the
// accumulator are read back only by the thread that wrote them.
template <int LG>
__global__ void __launch_bounds__(pair_threads<LG>(), pair_min_blocks<LG>())
k_corr_pair(const float *__restrict__ u, const float *__restrict__ dy, int Bt, int H, float *__restrict__ dK,
            float *__restrict__ dD, float2 *__restrict__ acc, float2 *__restrict__ zs) {
    constexpr int m = 1 << LG, L = m, T = pair_threads<LG>();
    constexpr int R0 = 1 << plan_lr(LG, 0), S0 = m / R0;
    constexpr int RL = 1 << plan_lr(LG, plan_P(LG) - 1), G = m / RL;
    extern __shared__ float2 sm[];
    const PairSmem s = pair_carve<LG>(sm);
    pair_tables<LG>(s);
    __syncthreads();
    const int nbp = (Bt + 1) / 2;
    for (int h = blockIdx.x; h < H; h += gridDim.x) {
        float4 *A0 = reinterpret_cast<float4 *>(acc + (size_t)h * 2 * m), *A1 = A0 + m / 2;
        float4 *Z0 = reinterpret_cast<float4 *>(zs + (size_t)h * 2 * m), *Z1 = Z0 + m / 2;
        for (int bp = 0; bp < nbp; ++bp) {
            const int b0 = 2 * bp;
            const bool has1 = b0 + 1 < Bt;
#pragma unroll 1
            for (int pass = 0; pass < 2; ++pass) {   // 0: u pair -> Zu; 1: dy pair -> acc
                const float *r0 = (pass == 0 ? u : dy) + ((size_t)b0 * H + h) * L;
                const float *r1 = r0 + (size_t)H * L;
                for (int j = threadIdx.x; j < S0; j += T) {
                    float2 v[R0];
                    static_for<0, R0>([&](auto p) {
                        const int k = j + p * S0;
                        v[p] = make_float2(__ldg(r0 + k), has1 ? __ldg(r1 + k) : 0.0f);
                    });
                    first_pass_halves<LG>(s, v, j);
                }
                __syncthreads();
                forward_middle_x2<LG, T>(s.b0, s.b1, s.tws);
                for (int g = threadIdx.x; g < G; g += T) {
                    const int base = g * RL, o = pidx(base);
                    float2 x[RL], z[RL];
                    load_contig<RL>(s.b0 + o, x);
                    load_contig<RL>(s.b1 + o, z);
                    dft<RL, -1>(x);
                    dft<RL, -1>(z);
                    static_for<0, RL / 2>([&](auto i) {
                        const int w = spec4_index<LG>(base, i);
                        const float2 x0 = x[2 * i], x1 = x[2 * i + 1], z0 = z[2 * i], z1 = z[2 * i + 1];
                        if (pass == 0) {
                            Z0[w] = make_float4(x0.x, x0.y, x1.x, x1.y);
                            Z1[w] = make_float4(z0.x, z0.y, z1.x, z1.y);
                        } else {
                            const float4 u0 = Z0[w], u1 = Z1[w];
                            const float2 p0 = cmulc(x0, make_float2(u0.x, u0.y));   // Zd conj(Zu)
                            const float2 p1 = cmulc(x1, make_float2(u0.z, u0.w));
                            const float2 q0 = cmulc(z0, make_float2(u1.x, u1.y));
                            const float2 q1 = cmulc(z1, make_float2(u1.z, u1.w));
                            float4 a0 = make_float4(p0.x, p0.y, p1.x, p1.y);
                            float4 a1 = make_float4(q0.x, q0.y, q1.x, q1.y);
                            if (bp > 0) {
                                const float4 c0 = A0[w], c1 = A1[w];
                                a0 = make_float4(a0.x + c0.x, a0.y + c0.y, a0.z + c0.z, a0.w + c0.w);
                                a1 = make_float4(a1.x + c1.x, a1.y + c1.y, a1.z + c1.z, a1.w + c1.w);
                            }
                            A0[w] = a0;
                            A1[w] = a1;
                        }
                    });
                }
                __syncthreads();   // the buffers are transformed again next
            }
        }
        // ---- inverse transform of the accumulated product, both halves
        for (int g = threadIdx.x; g < G; g += T) {
            const int base = g * RL, o = pidx(base);
            float2 x[RL], z[RL];
            static_for<0, RL / 2>([&](auto i) {
                const int w = spec4_index<LG>(base, i);
                const float4 c0 = A0[w], c1 = A1[w];
                x[2 * i] = make_float2(c0.x, c0.y);
                x[2 * i + 1] = make_float2(c0.z, c0.w);
                z[2 * i] = make_float2(c1.x, c1.y);
                z[2 * i + 1] = make_float2(c1.z, c1.w);
            });
            dft<RL, +1>(x);
            dft<RL, +1>(z);
            store_contig<RL>(s.b0 + o, x);
            store_contig<RL>(s.b1 + o, z);
        }
        __syncthreads();
        inverse_middle_x2<LG, T>(s.b0, s.b1, s.tws);
        const float scale = 1.0f / (float)(2 * m);
        float *dKh = dK + (size_t)h * L;
        last_pass_halves_sum<LG>(s, [&](int t, float2 r) {
            dKh[t] = r.x * scale;
            if (t == 0 && dD != nullptr) dD[h] = r.x * scale;
        });
        __syncthreads();   // the buffers are reused by the next channel
    }
}

namespace {
struct LaunchCache {
    int resident[64];
};
template <int LG>
cudaError_t run_corr(const float *u, const float *dy, int Bt, int H, float *dK, float *dD, void *ws,
                     cudaStream_t st) {
    static LaunchCache cache;
    constexpr int T = pair_threads<LG>();
    constexpr size_t smem = pair_smem_bytes<LG>(0);
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    int &res = cache.resident[dev & 63];
    if (res == 0) {
        e = cudaFuncSetAttribute(k_corr_pair<LG>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        int per_sm = 0, sms = 0;
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_corr_pair<LG>, T, smem);
        if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return e;
        if (per_sm * sms <= 0) return cudaErrorInvalidConfiguration;
        res = per_sm * sms;
    }
    const size_t half = corr_workspace_bytes(H, 1 << LG) / 2;
    float2 *acc = (float2 *)ws, *zs = (float2 *)((char *)ws + half);
    k_corr_pair<LG><<<res < H ? res : H, T, smem, st>>>(u, dy, Bt, H, dK, dD, acc, zs);
    return cudaGetLastError();
}
}  // namespace

size_t corr_workspace_bytes(int H, int L) {
    return 2 * (((size_t)H * 2 * L * sizeof(float2) + 255) & ~size_t(255));
}

cudaError_t launch_corr(const float *u, const float *dy, int Bt, int H, int L, float *dK, float *dD, void *ws,
                        cudaStream_t st) {
    switch (L) {
        case 16: return run_corr<4>(u, dy, Bt, H, dK, dD, ws, st);
        case 32: return run_corr<5>(u, dy, Bt, H, dK, dD, ws, st);
        case 64: return run_corr<6>(u, dy, Bt, H, dK, dD, ws, st);
        case 128: return run_corr<7>(u, dy, Bt, H, dK, dD, ws, st);
        case 256: return run_corr<8>(u, dy, Bt, H, dK, dD, ws, st);
        case 512: return run_corr<9>(u, dy, Bt, H, dK, dD, ws, st);
        case 1024: return run_corr<10>(u, dy, Bt, H, dK, dD, ws, st);
        case 2048: return run_corr<11>(u, dy, Bt, H, dK, dD, ws, st);
        case 4096: return run_corr<12>(u, dy, Bt, H, dK, dD, ws, st);
        case 8192: return run_corr<13>(u, dy, Bt, H, dK, dD, ws, st);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace s4
