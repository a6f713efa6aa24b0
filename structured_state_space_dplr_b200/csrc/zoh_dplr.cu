// zoh_dplr.cu -- zero-order hold of the full DPLR system ("The S4 kernel, from
// scratch", §3: the ZOH rule, here applied to the dense matrix
// A = diag(Lambda_f) - P_f Q_f^* of the conjugate-closed system):
//   Abar = exp(dt A),  Bbar = (integral_0^dt exp(A s) ds) B_f,  Cbar = C_f,
// and its truncated kernel K[k] = Re(C_f Abar^k Bbar), k < L. The §4
// generating-function shortcut (Cauchy sums at the roots of unity) belongs to
// the bilinear rule; under ZOH the kernel comes from dense powers instead.
//
// One CTA per channel, fp64 throughout, the state zero-padded to 64 (Nh <= 32;
// padded rows and columns of A are zero, so exp leaves an identity block there
// and Bbar, C_f are zero on it):
//  1. X = dt A / 2^s, bs = dt B_f / 2^s, with s the smallest count for which
//     ||X||_1 <= 1/2;
//  2. E = exp(X) and g = phi1(X) bs = sum_j X^j bs / (j + 1)! by Taylor
//     series of degree 16 in Horner form (together they are the top blocks of
//     exp([[X, bs], [0, 0]]); the truncation error is below 2^-17 / 17!);
//  3. s squarings of that augmented matrix: g <- E g + g, E <- E E.
//  The kernel: W[j] = Abar^j Bbar (j < 64), P = Abar^64 (six squarings),
//  r = C_f; for each block m of 64 steps K[64 m + j] = Re(r . W[j]), then
//  r <- r P.
#include "launch.h"
#include "s4dplr.h"

namespace s4 {

namespace zoh {
constexpr int kN = 64;           // padded state size
constexpr int kThreads = 256;
constexpr int kTaylor = 16;
constexpr size_t kMat = (size_t)kN * kN * sizeof(double2);   // 64 KB
// three matrices, six vectors, a [4][64] partial-sum array, scalars
constexpr size_t kSmem = 3 * kMat + 6 * kN * sizeof(double2) + 4 * kN * sizeof(double2) + 64;
}  // namespace zoh

namespace {

__device__ __forceinline__ double2 cfma(double2 a, double2 b, double2 c) {
    return make_double2(fma(a.x, b.x, fma(-a.y, b.y, c.x)), fma(a.x, b.y, fma(a.y, b.x, c.y)));
}
__device__ __forceinline__ double2 shfl_xor2(double2 v, int m) {
    return make_double2(__shfl_xor_sync(0xffffffffu, v.x, m), __shfl_xor_sync(0xffffffffu, v.y, m));
}

// Cm = scale (Am Bm) (+ I); 64 x 64 row-major, Cm distinct from Am and Bm.
// Thread (ty, tx) = (tid / 16, tid % 16) forms rows ty + 16 i, columns
// tx + 16 j (i, j < 4): Am reads are broadcasts, Bm reads 256 contiguous bytes.
__device__ void cmatmul(double2 *Cm, const double2 *Am, const double2 *Bm, double scale, bool ident) {
    using zoh::kN;
    const int ty = threadIdx.x >> 4, tx = threadIdx.x & 15;
    double2 acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = make_double2(0.0, 0.0);
#pragma unroll 2
    for (int k = 0; k < kN; ++k) {
        double2 a[4], b[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) a[i] = Am[(ty + 16 * i) * kN + k];
#pragma unroll
        for (int j = 0; j < 4; ++j) b[j] = Bm[k * kN + tx + 16 * j];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) acc[i][j] = cfma(a[i], b[j], acc[i][j]);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int r = ty + 16 * i, c = tx + 16 * j;
            double2 v = make_double2(scale * acc[i][j].x, scale * acc[i][j].y);
            if (ident && r == c) v.x += 1.0;
            Cm[r * kN + c] = v;
        }
}

// y = scale (A x) (+ add); y distinct from x. Row tid / 4, the 4 lanes of a
// row interleave over k.
__device__ void cmatvec(double2 *y, const double2 *A, const double2 *x, double scale, const double2 *add) {
    using zoh::kN;
    const int row = threadIdx.x >> 2, part = threadIdx.x & 3;
    double2 s = make_double2(0.0, 0.0);
#pragma unroll 4
    for (int it = 0; it < kN / 4; ++it) {
        const int k = part + 4 * it;
        s = cfma(A[row * kN + k], x[k], s);
    }
    s = make_double2(s.x + shfl_xor2(s, 1).x, s.y + shfl_xor2(s, 1).y);
    s = make_double2(s.x + shfl_xor2(s, 2).x, s.y + shfl_xor2(s, 2).y);
    if (part == 0) {
        double2 v = make_double2(scale * s.x, scale * s.y);
        if (add != nullptr) v = make_double2(v.x + add[row].x, v.y + add[row].y);
        y[row] = v;
    }
}

// y = x P (row vector times matrix), partial sums over four k ranges in part[4][64]
__device__ void cvecmat(double2 *y, const double2 *x, const double2 *Pm, double2 *part) {
    using zoh::kN;
    const int c = threadIdx.x & 63, q = threadIdx.x >> 6;
    double2 s = make_double2(0.0, 0.0);
#pragma unroll 4
    for (int k = 16 * q; k < 16 * q + 16; ++k) s = cfma(x[k], Pm[k * kN + c], s);
    part[q * kN + c] = s;
    __syncthreads();
    if (q == 0) {
        const double2 a = part[c], b = part[kN + c], d = part[2 * kN + c], e = part[3 * kN + c];
        y[c] = make_double2(a.x + b.x + d.x + e.x, a.y + b.y + d.y + e.y);
    }
}

// the channel's full-system entries: mode i < Nh stored, Nh <= i < 2 Nh its conjugate
__device__ __forceinline__ double2 full_mode(const float2 *v, int Nh, int i) {
    if (i < Nh) return make_double2(v[i].x, v[i].y);
    if (i < 2 * Nh) return make_double2(v[i - Nh].x, -v[i - Nh].y);
    return make_double2(0.0, 0.0);
}

}  // namespace

// MODE 0: write Abar [N, N], Bbar [N], Cfull [N]; MODE 1: write K [L]
template <int MODE>
__global__ void __launch_bounds__(zoh::kThreads, 1)
k_dplr_zoh(const float2 *__restrict__ Lambda, const float2 *__restrict__ P, const float2 *__restrict__ Q,
           const float2 *__restrict__ B, const float2 *__restrict__ C, const float *__restrict__ log_dt, int Nh,
           int L, float2 *__restrict__ Abar, float2 *__restrict__ Bbar, float2 *__restrict__ Cfull,
           float *__restrict__ K, unsigned *__restrict__ flags) {
    using zoh::kN;
    extern __shared__ __align__(16) unsigned char zsm[];
    double2 *M0 = reinterpret_cast<double2 *>(zsm);
    double2 *M1 = M0 + kN * kN, *M2 = M1 + kN * kN;
    double2 *v0 = M2 + kN * kN, *v1 = v0 + kN, *v2 = v1 + kN, *v3 = v2 + kN, *v4 = v3 + kN, *v5 = v4 + kN;
    double2 *part = v5 + kN;
    double *scal = reinterpret_cast<double *>(part + 4 * kN);
    int *iscal = reinterpret_cast<int *>(scal + 2);
    const int tid = threadIdx.x, h = blockIdx.x, N = 2 * Nh;
    const float2 *Lh = Lambda + (size_t)h * Nh, *Ph = P + (size_t)h * Nh, *Qh = Q + (size_t)h * Nh;
    const float2 *Bh = B + (size_t)h * Nh, *Ch = C + (size_t)h * Nh;
    const double dt = exp((double)log_dt[h]);

    // X = dt A (unscaled for now) in M0, bs = dt B_f in v0, C_f in v1
    for (int e = tid; e < kN * kN; e += zoh::kThreads) {
        const int r = e / kN, c = e % kN;
        const double2 p = full_mode(Ph, Nh, r), q = full_mode(Qh, Nh, c);
        // -(P_f[r] conj(Q_f[c])) + delta_rc Lambda_f[r]
        double2 v = make_double2(-(p.x * q.x + p.y * q.y), -(p.y * q.x - p.x * q.y));
        if (r == c) {
            const double2 l = full_mode(Lh, Nh, r);
            v.x += l.x;
            v.y += l.y;
        }
        M0[e] = make_double2(dt * v.x, dt * v.y);
    }
    if (tid < kN) {
        const double2 b = full_mode(Bh, Nh, tid);
        v0[tid] = make_double2(dt * b.x, dt * b.y);
        v1[tid] = full_mode(Ch, Nh, tid);
        if (flags != nullptr && tid < Nh && !(Lh[tid].x < 0.0f)) atomicOr(flags, S4_FLAG_UNSTABLE);
    }
    __syncthreads();
    // ||X||_1 = max column sum; s = squarings so that ||X / 2^s||_1 <= 1/2
    if (tid < kN) {
        double sum = 0.0;
        for (int r = 0; r < kN; ++r) sum += hypot(M0[r * kN + tid].x, M0[r * kN + tid].y);
        part[tid].x = sum;
    }
    __syncthreads();
    if (tid == 0) {
        double nrm = 0.0;
        for (int c = 0; c < kN; ++c) nrm = fmax(nrm, part[c].x);
        int s = 0;
        while (nrm > 0.5 && s < 64) {
            nrm *= 0.5;
            ++s;
        }
        iscal[0] = s;
        scal[0] = ldexp(1.0, -s);
    }
    __syncthreads();
    const int sq = iscal[0];
    const double sc = scal[0];
    for (int e = tid; e < kN * kN; e += zoh::kThreads) M0[e] = make_double2(sc * M0[e].x, sc * M0[e].y);
    if (tid < kN) v0[tid] = make_double2(sc * v0[tid].x, sc * v0[tid].y);
    // E = I in M1
    for (int e = tid; e < kN * kN; e += zoh::kThreads)
        M1[e] = make_double2((e / kN) == (e % kN) ? 1.0 : 0.0, 0.0);
    __syncthreads();
    // Horner: E <- I + X E / k, k = 16 .. 1
    double2 *E = M1, *T = M2;
    for (int k = zoh::kTaylor; k >= 1; --k) {
        cmatmul(T, M0, E, 1.0 / k, true);
        __syncthreads();
        double2 *t = E;
        E = T;
        T = t;
    }
    // g = phi1(X) bs: g <- bs + X g / k, k = 17 .. 2 (ping-pong v2 / v3)
    if (tid < kN) v2[tid] = v0[tid];
    __syncthreads();
    double2 *g = v2, *gn = v3;
    for (int k = zoh::kTaylor + 1; k >= 2; --k) {
        cmatvec(gn, M0, g, 1.0 / k, v0);
        __syncthreads();
        double2 *t = g;
        g = gn;
        gn = t;
    }
    // s squarings of the augmented matrix: g <- E g + g, E <- E E
    for (int i = 0; i < sq; ++i) {
        cmatvec(gn, E, g, 1.0, g);
        cmatmul(T, E, E, 1.0, false);
        __syncthreads();
        double2 *t = g;
        g = gn;
        gn = t;
        t = E;
        E = T;
        T = t;
    }
    // E = Abar, g = Bbar; M0 is free again
    if (MODE == 0) {
        float2 *Ao = Abar + (size_t)h * N * N;
        for (int e = tid; e < N * N; e += zoh::kThreads) {
            const double2 v = E[(e / N) * kN + e % N];
            Ao[e] = make_float2((float)v.x, (float)v.y);
        }
        if (tid < N) {
            Bbar[(size_t)h * N + tid] = make_float2((float)g[tid].x, (float)g[tid].y);
            Cfull[(size_t)h * N + tid] = make_float2((float)v1[tid].x, (float)v1[tid].y);
        }
        return;
    }
    // ---- kernel: P = Abar^64 by six squarings (T, M0 ping-pong), W in the third buffer
    double2 *Pa = T, *Pb = M0;
    cmatmul(Pa, E, E, 1.0, false);
    __syncthreads();
    for (int i = 0; i < 5; ++i) {
        cmatmul(Pb, Pa, Pa, 1.0, false);
        __syncthreads();
        double2 *t = Pa;
        Pa = Pb;
        Pb = t;
    }
    double2 *Pm = Pa, *W = Pb;   // Pm = Abar^64; W[j] = Abar^j Bbar (row j)
    if (tid < kN) W[tid] = g[tid];
    __syncthreads();
    for (int j = 1; j < kN; ++j) {
        cmatvec(W + j * kN, E, W + (j - 1) * kN, 1.0, nullptr);
        __syncthreads();
    }
    double2 *r = v4, *rn = v5;
    if (tid < kN) r[tid] = v1[tid];
    __syncthreads();
    float *Kh = K + (size_t)h * L;
    bool bad = false;
    const int nblk = (L + kN - 1) / kN;
    for (int m = 0; m < nblk; ++m) {
        {   // K[64 m + j] = Re(r . W[j]): row j = tid / 4, lanes of a row interleave over n
            const int j = tid >> 2, pq = tid & 3;
            double s = 0.0;
#pragma unroll 4
            for (int it = 0; it < kN / 4; ++it) {
                const int n = pq + 4 * it;
                s = fma(r[n].x, W[j * kN + n].x, fma(-r[n].y, W[j * kN + n].y, s));
            }
            s += __shfl_xor_sync(0xffffffffu, s, 1);
            s += __shfl_xor_sync(0xffffffffu, s, 2);
            const int k = m * kN + j;
            if (pq == 0 && k < L) {
                const float kv = (float)s;
                bad |= !isfinite(kv);
                Kh[k] = kv;
            }
        }
        if (m + 1 < nblk) {
            cvecmat(rn, r, Pm, part);
            __syncthreads();
            double2 *t = r;
            r = rn;
            rn = t;
        }
    }
    if (flags != nullptr && bad) atomicOr(flags, S4_FLAG_NONFINITE);
}

cudaError_t launch_dplr_zoh(const float2 *Lambda, const float2 *P, const float2 *Q, const float2 *B,
                            const float2 *C, const float *log_dt, int H, int Nh, int L, float2 *Abar,
                            float2 *Bbar, float2 *Cfull, float *K, unsigned *flags, cudaStream_t st) {
    static bool attr_set[64][2];   // per device and mode; setting the attribute twice is harmless
    const int mode = K != nullptr ? 1 : 0;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (!attr_set[dev & 63][mode]) {
        e = cudaFuncSetAttribute(mode ? k_dplr_zoh<1> : k_dplr_zoh<0>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)zoh::kSmem);
        if (e != cudaSuccess) return e;
        attr_set[dev & 63][mode] = true;
    }
    if (mode)
        k_dplr_zoh<1><<<H, zoh::kThreads, zoh::kSmem, st>>>(Lambda, P, Q, B, C, log_dt, Nh, L, nullptr, nullptr,
                                                             nullptr, K, flags);
    else
        k_dplr_zoh<0><<<H, zoh::kThreads, zoh::kSmem, st>>>(Lambda, P, Q, B, C, log_dt, Nh, 0, Abar, Bbar, Cfull,
                                                             nullptr, nullptr);
    return cudaGetLastError();
}

}  // namespace s4
