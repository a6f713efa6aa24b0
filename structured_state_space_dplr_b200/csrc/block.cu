// block.cu -- the S4Block around the S4 layer ("The S4 kernel, from
// scratch", §6 "Trainable layer": a pre-norm, a GLU-gated projection and a
// residual connection):
//
//   z   = LayerNorm_h(x) * gamma + beta           (over the H channels at each (b, t))
//   y   = K * z + D z                             (the S4 layer, spectral.cu)
//   p   = W y + bias,  W [2H, H]                  (at each (b, t))
//   out = x + p[:H] * sigmoid(p[H:])
//
// The projection is a dense contraction over channels and runs on the tensor
// cores. Per CTA: one batch row b, 64 output channels and N (<= 128) time
// steps; the 64 value rows and the 64 gate rows of W are interleaved into the
// 128 rows of the MMA's A operand (row 2i = value of channel i, row 2i + 1 =
// its gate), so the epilogue pairs them with one lane exchange. Operands are
// fp32 split into bf16 high and low parts, and the three products
// A_hi B_hi + A_hi B_lo + A_lo B_hi are accumulated in fp32 in tensor memory
// (the dropped A_lo B_lo and the split residues are ~2^-17 relative). W is
// split once into the MMA's shared-memory image by s4_glu_projection_prepare;
// y is split on the way into shared memory, 32 channels per stage, two
// stages in flight.
#include <cuda_bf16.h>

#include "launch.h"
#include "s4dplr.h"
#include "umma.cuh"

namespace s4 {

namespace glu {
constexpr int kRows = 128;                   // MMA M: 64 output channels x (value, gate)
constexpr int kOut = kRows / 2;
constexpr int kKc = 32;                      // channels per stage (two K = 16 MMA steps)
constexpr int kNmax = 128;                   // time steps per tile (MMA N)
constexpr int kThreads = 256;
constexpr int kAImg = kRows * kKc * 2;       // bytes of one bf16 operand image of W (8 KB)
constexpr int kBImg = kNmax * kKc * 2;       // bytes of one bf16 operand image of y (8 KB)
constexpr int kStage = 2 * kAImg + 2 * kBImg;   // A hi, A lo, B hi, B lo
constexpr int kStages = 2;
constexpr int kTmemCols = 128;
constexpr size_t kSmem = (size_t)kStages * kStage + 64;
constexpr uint32_t kSpinLimit = 1u << 24;
static_assert(kOut * (kNmax + 1) * 4 <= kStages * kStage, "epilogue tile must fit in the stage buffers");
}  // namespace glu

__host__ __device__ inline int glu_nob(int H) { return (H + glu::kOut - 1) / glu::kOut; }
__host__ __device__ inline int glu_nkc(int H) { return (H + glu::kKc - 1) / glu::kKc; }

size_t glu_workspace_bytes(int H) { return (size_t)glu_nob(H) * glu_nkc(H) * 2 * glu::kAImg; }

namespace {

// byte offset of element (r, k) in a K-major bf16 tile of `rows` rows
__device__ __forceinline__ int kmajor_off(int rows, int r, int k) {
    return (r & 7) * 16 + (r >> 3) * 128 + (k >> 3) * (rows / 8) * 128 + (k & 7) * 2;
}

// 8 floats -> 8 bf16 high parts and 8 bf16 low parts (v - hi), packed
__device__ __forceinline__ void split8(const float (&v)[8], uint4 &hi, uint4 &lo) {
    uint32_t h[4], l[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const __nv_bfloat162 hp = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
        const float r0 = v[2 * i] - __low2float(hp), r1 = v[2 * i + 1] - __high2float(hp);
        const __nv_bfloat162 lp = __floats2bfloat162_rn(r0, r1);
        h[i] = *reinterpret_cast<const uint32_t *>(&hp);
        l[i] = *reinterpret_cast<const uint32_t *>(&lp);
    }
    hi = make_uint4(h[0], h[1], h[2], h[3]);
    lo = make_uint4(l[0], l[1], l[2], l[3]);
}

__device__ __forceinline__ float sigmoidf_(float g) { return 1.0f / (1.0f + __expf(-g)); }

}  // namespace

// ---------------------------------------------------------------- layer norm
// One CTA: 32 consecutive time steps of one batch row; warp w sums channels
// w, w + 8, ... (a warp reads 128 contiguous bytes per channel). The sums are
// taken about x[b, 0, t] (shifted data: no cancellation for large means).
// z may be x (in place): every element is read and then written by one thread.
__global__ void __launch_bounds__(256) k_layernorm_channels(const float *x, const float *__restrict__ gamma,
                                                            const float *__restrict__ beta, float eps, int H,
                                                            int L, float *z) {
    __shared__ float s1[8][33], s2[8][33], mu_s[32], rs_s[32];
    const int tl = threadIdx.x & 31, hs = threadIdx.x >> 5;
    const int t = blockIdx.x * 32 + tl;
    const bool in = t < L;
    const size_t base = (size_t)blockIdx.y * H * L + t;
    const float c = in ? x[base] : 0.0f;
    float a1 = 0.0f, a2 = 0.0f;
    if (in) {
#pragma unroll 4
        for (int h = hs; h < H; h += 8) {
            const float d = x[base + (size_t)h * L] - c;
            a1 += d;
            a2 = fmaf(d, d, a2);
        }
    }
    s1[hs][tl] = a1;
    s2[hs][tl] = a2;
    __syncthreads();
    if (hs == 0) {
        float S1 = 0.0f, S2 = 0.0f;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            S1 += s1[i][tl];
            S2 += s2[i][tl];
        }
        const float m1 = S1 / (float)H;
        const float var = fmaxf(S2 / (float)H - m1 * m1, 0.0f);
        mu_s[tl] = c + m1;
        rs_s[tl] = rsqrtf(var + eps);
    }
    __syncthreads();
    if (!in) return;
    const float mu = mu_s[tl], rs = rs_s[tl];
#pragma unroll 4
    for (int h = hs; h < H; h += 8) {
        const size_t o = base + (size_t)h * L;
        z[o] = (x[o] - mu) * rs * __ldg(gamma + h) + __ldg(beta + h);
    }
}

// ------------------------------------------------------- W -> operand images
// Image (ob, c) holds rows 2i / 2i + 1 = W[64 ob + i] / W[H + 64 ob + i],
// columns h = 32 c .. 32 c + 31, as bf16 high part (first kAImg bytes) and
// low part (next kAImg bytes); rows and columns past H are zero. One thread
// writes 8 columns of one row.
__global__ void k_glu_prepare(const float *__restrict__ W, int H, unsigned char *__restrict__ img) {
    using namespace glu;
    const int nkc = glu_nkc(H);
    const long long total = (long long)glu_nob(H) * nkc * kRows * (kKc / 8);
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= total) return;
    const int q = (int)(i % (kKc / 8));
    const int r = (int)((i / (kKc / 8)) % kRows);
    const long long oc = i / ((kKc / 8) * kRows);
    const int c = (int)(oc % nkc), ob = (int)(oc / nkc);
    const int o = ob * kOut + (r >> 1);
    const size_t wrow = (size_t)((r & 1) ? H + o : o) * H;
    float v[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const int h = c * kKc + 8 * q + j;
        v[j] = (o < H && h < H) ? W[wrow + h] : 0.0f;
    }
    uint4 hi, lo;
    split8(v, hi, lo);
    unsigned char *base = img + (size_t)oc * 2 * kAImg + kmajor_off(kRows, r, 8 * q);
    *reinterpret_cast<uint4 *>(base) = hi;
    *reinterpret_cast<uint4 *>(base + kAImg) = lo;
}

// ------------------------------------------- projection + GLU + residual
__global__ void __launch_bounds__(glu::kThreads, 1)
k_glu_projection_tc(const float *__restrict__ y, const float *x, const float *__restrict__ bias,
                    const unsigned char *__restrict__ img, int H, int L, int N, float *out,
                    unsigned *__restrict__ flags) {
    using namespace glu;
    extern __shared__ __align__(1024) unsigned char sm[];
    uint64_t *mbar = reinterpret_cast<uint64_t *>(sm + kStages * kStage);   // [2]
    uint32_t *tslot = reinterpret_cast<uint32_t *>(mbar + 2);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nob = glu_nob(H), nkc = glu_nkc(H), ntt = L / N;
    int item = blockIdx.x;
    const int ob = item % nob;
    item /= nob;
    const int tt = item % ntt, b = item / ntt;
    const int t0 = tt * N;

    if (tid == 0) {
        umma::mbar_init(&mbar[0], 1);
        umma::mbar_init(&mbar[1], 1);
        umma::fence_mbar_init();
    }
    if (warp == 0) umma::tmem_alloc(tslot, kTmemCols);
    umma::fence_before_sync();
    __syncthreads();
    umma::fence_after_sync();
    const uint32_t tmem = *tslot;
    const uint32_t id = umma::idesc(1, kRows, N);
    const uint32_t b_lbo = (uint32_t)(N / 8) * 128, a_lbo = (kRows / 8) * 128;

    const float *yb = y + (size_t)b * H * L + t0;
    const int tl = tid & (kNmax - 1), kg = tid >> 7;   // B-tile row (time step) and channel group
    uint32_t ph = 0u;   // bit s: parity of the next completion of mbar[s]
    bool ok = true;
    for (int c = 0; c < nkc; ++c) {
        const int s = c & 1;
        unsigned char *stage = sm + s * kStage;
        if (c >= 2) {   // the MMAs of chunk c - 2 read this stage: wait for them
            const bool done = tid != 0 || umma::mbar_wait(&mbar[s], (ph >> s) & 1u, kSpinLimit);
            ph ^= 1u << s;
            ok = __syncthreads_and(done) != 0;
            if (!ok) break;
        }
        // A: the prepared image of W for (ob, c), hi then lo, 16 bytes per copy
        const unsigned char *src = img + ((size_t)ob * nkc + c) * 2 * kAImg;
#pragma unroll
        for (int i = 0; i < (2 * kAImg) / 16 / kThreads; ++i) {
            const int j = tid + i * kThreads;
            umma::cp_async16(stage + 16 * j, src + 16 * j);
        }
        umma::cp_async_commit();
        // B: y[b, 32 c + 8 q + j, t0 + tl] for groups q = kg, kg + 2, split
        if (tl < N) {
#pragma unroll
            for (int qq = 0; qq < 2; ++qq) {
                const int q = kg + 2 * qq;
                float v[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const int h = c * kKc + 8 * q + j;
                    v[j] = h < H ? __ldg(yb + (size_t)h * L + tl) : 0.0f;
                }
                uint4 hi, lo;
                split8(v, hi, lo);
                unsigned char *bt = stage + 2 * kAImg + kmajor_off(N, tl, 8 * q);
                *reinterpret_cast<uint4 *>(bt) = hi;
                *reinterpret_cast<uint4 *>(bt + kBImg) = lo;
            }
        }
        umma::cp_async_wait_all();
        umma::fence_proxy_async();
        umma::fence_before_sync();
        __syncthreads();
        if (tid == 0) {
            umma::fence_after_sync();
            const uint32_t Ah = umma::saddr(stage), Al = Ah + kAImg;
            const uint32_t Bh = Ah + 2 * kAImg, Bl = Bh + kBImg;
            const uint32_t As[3] = {Ah, Ah, Al}, Bs[3] = {Bh, Bl, Bh};
#pragma unroll
            for (int pr = 0; pr < 3; ++pr) {
#pragma unroll
                for (int kk = 0; kk < kKc / 16; ++kk) {
                    const uint64_t da = umma::smem_desc(As[pr] + kk * 2 * a_lbo, a_lbo);
                    const uint64_t db = umma::smem_desc(Bs[pr] + kk * 2 * b_lbo, b_lbo);
                    umma::mma_bf16(tmem, da, db, id, c > 0 || pr > 0 || kk > 0);
                }
            }
            umma::commit(&mbar[s]);
        }
    }
    if (ok) {   // the last chunk's commit covers every MMA; also drain the other stage's
        const int sl = (nkc - 1) & 1;
        bool done = true;
        if (tid == 0) {
            done = umma::mbar_wait(&mbar[sl], (ph >> sl) & 1u, kSpinLimit);
            if (done && nkc >= 2) done = umma::mbar_wait(&mbar[sl ^ 1], (ph >> (sl ^ 1)) & 1u, kSpinLimit);
        }
        ok = __syncthreads_and(done) != 0;
    }
    if (!ok && tid == 0 && flags != nullptr) atomicOr(flags, S4_FLAG_TIMEOUT);
    umma::fence_after_sync();

    if (ok) {
        // read back: warp w owns rows 32 (w % 4) + lane (row 2i value / 2i + 1
        // gate of channel 64 ob + i) and the 16-column groups g = w / 4 (mod 2)
        float *tile = reinterpret_cast<float *>(sm);   // [64][N + 1], over the stage buffers
        const int q4 = warp & 3, row = 32 * q4 + lane, ol = row >> 1;
        const bool gate_row = row & 1;
        const int o = ob * kOut + ol;
        const float bv = o < H ? __ldg(bias + o) : 0.0f, bg = o < H ? __ldg(bias + H + o) : 0.0f;
        for (int g = warp >> 2; g < N / 16; g += 2) {
            uint32_t v[16];
            umma::ld_32x32b_x16(tmem + ((uint32_t)(32 * q4) << 16) + (uint32_t)(16 * g), v);
            float r[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const float mine = __uint_as_float(v[i]);
                const float other = __shfl_xor_sync(0xffffffffu, mine, 1);
                const float val = gate_row ? other : mine, gt = gate_row ? mine : other;
                r[i] = (val + bv) * sigmoidf_(gt + bg);
            }
            // the value lane stores columns 0..7 of the group, the gate lane 8..15
            const int i0 = gate_row ? 8 : 0;
#pragma unroll
            for (int i = 0; i < 8; ++i) tile[ol * (N + 1) + 16 * g + i0 + i] = gate_row ? r[8 + i] : r[i];
        }
    }
    umma::fence_before_sync();
    __syncthreads();
    if (ok) {
        const size_t ob_base = ((size_t)b * H + (size_t)ob * kOut) * L + t0;
        const float *tile = reinterpret_cast<const float *>(sm);
        for (int i = tid; i < kOut * N; i += kThreads) {
            const int ol = i / N, t = i - ol * N;
            if (ob * kOut + ol >= H) break;
            const size_t gi = ob_base + (size_t)ol * L + t;
            out[gi] = x[gi] + tile[ol * (N + 1) + t];   // out may be x: read, then written, by this thread
        }
    }
    if (warp == 0) umma::tmem_dealloc(tmem, kTmemCols);
}

// ------------------------------------------------------------------ launchers
cudaError_t launch_layernorm_channels(const float *x, const float *gamma, const float *beta, float eps, int Bt,
                                      int H, int L, float *z, cudaStream_t st) {
    dim3 grid((L + 31) / 32, Bt);
    k_layernorm_channels<<<grid, 256, 0, st>>>(x, gamma, beta, eps, H, L, z);
    return cudaGetLastError();
}

cudaError_t launch_glu_prepare(const float *W, int H, void *ws, cudaStream_t st) {
    const long long total = (long long)glu_nob(H) * glu_nkc(H) * glu::kRows * (glu::kKc / 8);
    k_glu_prepare<<<(unsigned)((total + 255) / 256), 256, 0, st>>>(W, H, static_cast<unsigned char *>(ws));
    return cudaGetLastError();
}

cudaError_t launch_glu_projection(const float *y, const float *x, const float *bias, const void *ws, int Bt, int H,
                                  int L, float *out, unsigned *flags, cudaStream_t st) {
    static bool attr_set = false;   // per function; setting it twice is harmless
    if (!attr_set) {
        cudaError_t e = cudaFuncSetAttribute(k_glu_projection_tc, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)glu::kSmem);
        if (e != cudaSuccess) return e;
        attr_set = true;
    }
    const int N = L < glu::kNmax ? L : glu::kNmax;
    const long long items = (long long)Bt * glu_nob(H) * (L / N);
    k_glu_projection_tc<<<(unsigned)items, glu::kThreads, glu::kSmem, st>>>(
        y, x, bias, static_cast<const unsigned char *>(ws), H, L, N, out, flags);
    return cudaGetLastError();
}

}  // namespace s4
