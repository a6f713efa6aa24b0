// s4d.cu -- diagonal S4D with zero-order hold ("S4" wiki page, section
// "S4D"; ZOH rule of "The S4 kernel, from scratch", §3):
//   Abar_n = exp(dt a_n),  Bbar_n = (exp(dt a_n) - 1)/a_n B_n,
//   K[h, k] = 2 Re sum_n C_n Bbar_n Abar_n^k   (truncated, k < L).
//
// Vandermonde kernel: with k = kh KB + kl,
//   Abar^k = Abar^(kh KB) Abar^kl,  so
//   K[h, kh KB + kl] = 2 sum_n Re( G[n, kh] T[n, kl] ),
//   G[n, kh] = C_n Bbar_n Abar_n^(kh KB),  T[n, kl] = Abar_n^kl,
// i.e. two FMAs per (k, n) term once the two small tables are in shared
// memory. Each table entry is built from its own exponent with an fp64 phase
// reduction -- the phase k dt Im(a) reaches ~1e5 rad, far beyond what an fp32
// product can resolve -- then evaluated with fp32 sincospif / expf.
#include "common.cuh"
#include "launch.h"
#include "s4dplr.h"

namespace s4 {

// exp(x) - 1 for complex x without cancellation: the real part is
// expm1(xr) cos(xi) - 2 sin^2(xi/2).
__device__ __forceinline__ double2 cexpm1_d(double xr, double xi) {
    double s, c, sh, ch;
    sincos(xi, &s, &c);
    sincos(0.5 * xi, &sh, &ch);
    const double em = expm1(xr);
    return make_double2(em * c - 2.0 * sh * sh, (em + 1.0) * s);
}

struct ZohMode {
    double2 abar;      // exp(dt a)
    double2 bbar;      // (exp(dt a) - 1)/a * B
    double kre;        // dt Re(a)    (log-magnitude per step)
    double kph;        // dt Im(a) / (2 pi)  (turns per step)
};

__device__ __forceinline__ ZohMode zoh_mode(float2 a, float2 b, double dt) {
    ZohMode z;
    const double ar = a.x, ai = a.y;
    const double xr = dt * ar, xi = dt * ai;
    double s, c;
    sincos(xi, &s, &c);
    const double e = exp(xr);
    z.abar = make_double2(e * c, e * s);
    double2 ratio;   // (exp(x) - 1)/a
    if (fabs(xr) + fabs(xi) < 1e-4) {   // dt (1 + x/2 + x^2/6 + x^3/24)
        const double x2r = xr * xr - xi * xi, x2i = 2 * xr * xi;
        const double x3r = x2r * xr - x2i * xi, x3i = x2r * xi + x2i * xr;
        ratio = make_double2(dt * (1.0 + xr / 2 + x2r / 6 + x3r / 24), dt * (xi / 2 + x2i / 6 + x3i / 24));
    } else {
        const double2 em = cexpm1_d(xr, xi);
        const double d = ar * ar + ai * ai;
        ratio = make_double2((em.x * ar + em.y * ai) / d, (em.y * ar - em.x * ai) / d);
    }
    z.bbar = make_double2(ratio.x * b.x - ratio.y * b.y, ratio.x * b.y + ratio.y * b.x);
    z.kre = xr;
    z.kph = xi * 0.15915494309189533577;   // 1/(2 pi)
    return z;
}

// Abar^e in fp32 with an fp64 phase reduction
__device__ __forceinline__ float2 zoh_power(const ZohMode &z, int e) {
    double ph = (double)e * z.kph;
    ph -= rint(ph);
    float s, c;
    sincospif(2.0f * (float)ph, &s, &c);
    const float mag = expf((float)((double)e * z.kre));
    return make_float2(mag * c, mag * s);
}

constexpr int kVdmThreads = 256;
constexpr int kVdmKB = 64;      // kl range
constexpr int kVdmKH = 128;     // kh per block
constexpr int kVdmModes = 32;   // modes per shared-memory chunk
constexpr int kVdmTH = 4, kVdmTL = 8;   // per-thread output tile (kh x kl)

__global__ void __launch_bounds__(kVdmThreads)
k_vandermonde(const float2 *__restrict__ A, const float2 *__restrict__ B, const float2 *__restrict__ Cc,
              const float *__restrict__ log_dt, int Nh, int L, float *__restrict__ K,
              unsigned *__restrict__ flags) {
    extern __shared__ double vdm_smem[];   // kph[M] | kre[M] | G[M][KH] | T[M][KB] | CB[M]
    double *sKph = vdm_smem, *sKre = vdm_smem + kVdmModes;
    float2 (*sG)[kVdmKH] = reinterpret_cast<float2 (*)[kVdmKH]>(vdm_smem + 2 * kVdmModes);
    float2 (*sT)[kVdmKB] = reinterpret_cast<float2 (*)[kVdmKB]>(&sG[kVdmModes][0]);
    float2 *sCB = &sT[kVdmModes][0];
    const int h = blockIdx.y;
    const int KB = L < kVdmKB ? L : kVdmKB;
    const int nkh = L / KB;
    const int kh0 = blockIdx.x * kVdmKH;
    const int khc = (nkh - kh0) < kVdmKH ? (nkh - kh0) : kVdmKH;
    const double dt = exp((double)__ldg(log_dt + h));
    const int nlg = KB / kVdmTL;                 // kl groups
    const int ntiles = ((khc + kVdmTH - 1) / kVdmTH) * nlg;   // <= 256
    const int my = threadIdx.x;                  // one output tile per thread
    const int khb = (my / nlg) * kVdmTH, klb = (my % nlg) * kVdmTL;
    float acc[kVdmTH][kVdmTL];
#pragma unroll
    for (int a = 0; a < kVdmTH; ++a)
#pragma unroll
        for (int b = 0; b < kVdmTL; ++b) acc[a][b] = 0.0f;

    {
        for (int n0 = 0; n0 < Nh; n0 += kVdmModes) {
            const int nc = (Nh - n0) < kVdmModes ? (Nh - n0) : kVdmModes;
            __syncthreads();
            for (int n = threadIdx.x; n < nc; n += kVdmThreads) {
                const size_t o = (size_t)h * Nh + n0 + n;
                const float2 an = A[o];
                const ZohMode z = zoh_mode(an, B[o], dt);
                const float2 cn = Cc[o];
                sKre[n] = z.kre;
                sKph[n] = z.kph;
                sCB[n] = make_float2((float)(cn.x * z.bbar.x - cn.y * z.bbar.y),
                                     (float)(cn.x * z.bbar.y + cn.y * z.bbar.x));
                if (flags != nullptr && blockIdx.x == 0 && !(an.x < 0.0f)) atomicOr(flags, S4_FLAG_UNSTABLE);
            }
            __syncthreads();
            for (int i = threadIdx.x; i < nc * (kVdmKB + kVdmKH); i += kVdmThreads) {
                const int n = i / (kVdmKB + kVdmKH), r = i % (kVdmKB + kVdmKH);
                ZohMode z;
                z.kre = sKre[n];
                z.kph = sKph[n];
                if (r < kVdmKB) {
                    if (r < KB) sT[n][r] = zoh_power(z, r);
                } else {
                    const int kh = r - kVdmKB;
                    if (kh < khc) sG[n][kh] = cmul(sCB[n], zoh_power(z, (kh0 + kh) * KB));
                }
            }
            __syncthreads();
            if (my < ntiles) {
                for (int n = 0; n < nc; ++n) {
                    float2 g[kVdmTH], t[kVdmTL];
#pragma unroll
                    for (int a = 0; a < kVdmTH; ++a) g[a] = sG[n][(khb + a) < khc ? khb + a : 0];
#pragma unroll
                    for (int b = 0; b < kVdmTL; ++b) t[b] = sT[n][klb + b];
#pragma unroll
                    for (int a = 0; a < kVdmTH; ++a)
#pragma unroll
                        for (int b = 0; b < kVdmTL; ++b)
                            acc[a][b] = fmaf(g[a].x, t[b].x, fmaf(-g[a].y, t[b].y, acc[a][b]));
                }
            }
        }
    }
    if (my < ntiles) {
        bool bad = false;
#pragma unroll
        for (int a = 0; a < kVdmTH; ++a) {
            if (khb + a < khc) {
                float *out = K + (size_t)h * L + (size_t)(kh0 + khb + a) * KB + klb;
#pragma unroll
                for (int b = 0; b < kVdmTL; b += 4) {
                    const float4 v = make_float4(2.f * acc[a][b], 2.f * acc[a][b + 1],
                                                 2.f * acc[a][b + 2], 2.f * acc[a][b + 3]);
                    bad |= !(isfinite(v.x) && isfinite(v.y) && isfinite(v.z) && isfinite(v.w));
                    *reinterpret_cast<float4 *>(out + b) = v;
                }
            }
        }
        if (bad && flags != nullptr) atomicOr(flags, S4_FLAG_NONFINITE);
    }
}

__global__ void k_s4d_zoh(const float2 *__restrict__ A, const float2 *__restrict__ B,
                          const float *__restrict__ log_dt, int H, int Nh,
                          float2 *__restrict__ Abar, float2 *__restrict__ Bbar) {
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= (long long)H * Nh) return;
    const int h = (int)(i / Nh);
    const ZohMode z = zoh_mode(A[i], B[i], exp((double)__ldg(log_dt + h)));
    Abar[i] = make_float2((float)z.abar.x, (float)z.abar.y);
    Bbar[i] = make_float2((float)z.bbar.x, (float)z.bbar.y);
}

cudaError_t launch_vandermonde(const float2 *A, const float2 *B, const float2 *C, const float *log_dt,
                               int H, int Nh, int L, float *K, unsigned *flags, cudaStream_t st) {
    const int KB = L < kVdmKB ? L : kVdmKB;
    const int nkh = L / KB;
    dim3 grid((nkh + kVdmKH - 1) / kVdmKH, H);
    constexpr size_t smem = 2 * kVdmModes * sizeof(double) +
                            (size_t)kVdmModes * (kVdmKH + kVdmKB + 1) * sizeof(float2);
    static bool attr_set = false;   // the attribute is per function; setting it twice is harmless
    if (!attr_set) {
        cudaError_t e = cudaFuncSetAttribute(k_vandermonde, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        attr_set = true;
    }
    k_vandermonde<<<grid, kVdmThreads, smem, st>>>(A, B, C, log_dt, Nh, L, K, flags);
    return cudaGetLastError();
}

cudaError_t launch_s4d_zoh(const float2 *A, const float2 *B, const float *log_dt, int H, int Nh,
                           float2 *Abar, float2 *Bbar, cudaStream_t st) {
    const long long n = (long long)H * Nh;
    k_s4d_zoh<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(A, B, log_dt, H, Nh, Abar, Bbar);
    return cudaGetLastError();
}

}  // namespace s4
