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
// cores: D[t, n] = sum_h y[b, h, t0 + t] W'[n, h], one tile = 128 time steps
// (the MMA's M, tensor-memory lanes) x 256 rows of W' (the MMA's N), where W'
// interleaves the value and gate rows of 128 output channels (row 2i = value
// of channel i, row 2i + 1 = its gate), so one thread holds both halves of a
// GLU. Operands are fp32 split into bf16 high and low parts, and the three
// products y_hi W_hi + y_hi W_lo + y_lo W_hi are accumulated in fp32 in
// tensor memory (the dropped y_lo W_lo and the split residues are ~2^-17
// relative). W is split once into the MMA's shared-memory image by
// s4_glu_projection_prepare.
//
// The kernel is persistent (one CTA per SM) and warp-specialized:
//   warp 0      loader: TMA of raw fp32 y chunks [32 channels x 128 steps]
//               and bulk copies of the W image chunks, into rings;
//   warps 1-4   split each raw y chunk into the bf16 image of the operand;
//   warp 5      one thread issues the MMAs (6 per chunk) and the commits;
//   warp 6      x loader: TMA of the residual x in [32 channels x 128 steps]
//               chunks, into a ring;
//   warps 7-14  epilogue: tensor memory -> GLU + bias + residual -> out; two
//               warps per tensor-memory lane quadrant, each half the columns.
// The accumulator is double-buffered (2 x 256 of the 512 tensor-memory
// columns), so the epilogue of one tile overlaps the MMAs of the next. Every
// wait is bounded: on expiry the CTA sets S4_FLAG_TIMEOUT, every role stops,
// copies in flight are waited for (bounded) and tensor memory is freed.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>

#include <mutex>

#include "launch.h"
#include "s4dplr.h"
#include "umma.cuh"

namespace s4 {

namespace glu {
constexpr int kTm = 128;                      // MMA M: time steps per tile
constexpr int kNr = 256;                      // MMA N: rows of W' per tile
constexpr int kCh = kNr / 2;                  // output channels per tile
constexpr int kKc = 32;                       // contraction channels per chunk (two K = 16 steps)
constexpr int kYImg = kTm * kKc * 2;          // 8 KB: one bf16 image of a y chunk
constexpr int kWImg = kNr * kKc * 2;          // 16 KB: one bf16 image of a W' chunk
constexpr int kStage = 2 * kYImg + 2 * kWImg; // 48 KB: y hi, y lo, W hi, W lo
constexpr int kRawBytes = kKc * kTm * 4;      // 16 KB: a raw fp32 chunk [32][<= 128]
constexpr int kXc = 32;                       // output channels per x chunk of the epilogue
constexpr int kS = 3, kR = 3, kX = 2;         // operand stages, raw y ring, x ring
constexpr int kOffRaw = kS * kStage;
constexpr int kOffX = kOffRaw + kR * kRawBytes;
constexpr int kOffBar = kOffX + kX * kRawBytes;
constexpr int kNumBars = 2 * kR + 3 * kS + 2 + 2 + 2 * kX;
constexpr size_t kSmem = (size_t)kOffBar + kNumBars * 8 + 16;
// warps: 0 y/W loader, 1-4 converters, 5 MMA, 6 x loader, 7-14 epilogue
constexpr int kThreads = 15 * 32;
constexpr int kEpiWarp0 = 7, kEpiThreads = 256;
constexpr int kTmemCols = 512;
constexpr uint32_t kSpinLimit = 1u << 22;
static_assert(kSmem <= 232448, "shared memory per CTA");
}  // namespace glu

__host__ __device__ inline int glu_nnb(int H) { return (H + glu::kCh - 1) / glu::kCh; }
__host__ __device__ inline int glu_nkc(int H) { return (H + glu::kKc - 1) / glu::kKc; }

size_t glu_workspace_bytes(int H) { return (size_t)glu_nkc(H) * glu_nnb(H) * 2 * glu::kWImg; }

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

// logistic function; __expf and __fdividef keep it to a few instructions
// (relative error ~1e-7, far below the projection's)
__device__ __forceinline__ float sigmoidf_(float g) { return __fdividef(1.0f, 1.0f + __expf(-g)); }

// ---- asynchronous copies and barrier arrivals (inline PTX)
__device__ __forceinline__ void arrive(uint64_t *m) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(umma::saddr(m)) : "memory");
}
__device__ __forceinline__ void arrive_expect_tx(uint64_t *m, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(umma::saddr(m)), "r"(bytes)
                 : "memory");
}
// 3-D tiled TMA load of the box at (x, y, z) into this CTA's shared memory only
__device__ __forceinline__ void tma_load_3d(void *dst, const CUtensorMap *map, int x, int y, int z, uint64_t *m) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], "
        "[%5];" ::"r"(umma::saddr(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(umma::saddr(m))
        : "memory");
}
// contiguous bulk copy global -> this CTA's shared memory; 16-byte aligned, size % 16 == 0
__device__ __forceinline__ void bulk_load(void *dst, const void *src, uint32_t bytes, uint64_t *m) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     umma::saddr(dst)),
                 "l"(src), "r"(bytes), "r"(umma::saddr(m))
                 : "memory");
}
__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap *map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}
__device__ __forceinline__ void named_sync(int id, int threads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}
// AND of p over the `threads` threads of named barrier `id` (all of them get it)
__device__ __forceinline__ bool named_and(int id, int threads, bool p) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred q, o;\n\tsetp.ne.u32 q, %1, 0;\n\tbar.red.and.pred o, %2, %3, q;\n\t"
        "selp.u32 %0, 1, 0, o;\n\t}\n"
        : "=r"(r)
        : "r"((uint32_t)p), "r"(id), "r"(threads)
        : "memory");
    return r != 0;
}

// the per-CTA tile sequence: tile i = ((b * ntt + tt) * nnb + nb), channel
// block fastest (the tiles that read the same y chunks run side by side)
struct Tile {
    int b, t0, nb;
};
__device__ __forceinline__ Tile tile_of(long long i, int nnb, int ntt, int N) {
    Tile t;
    t.nb = (int)(i % nnb);
    const long long r = i / nnb;
    t.t0 = (int)(r % ntt) * N;
    t.b = (int)(r / ntt);
    return t;
}
// x chunks of a tile: 32 output channels each, up to H
__device__ __forceinline__ int x_chunks(int H, int nb) {
    const int left = H - nb * glu::kCh;
    const int n = (left + glu::kXc - 1) / glu::kXc;
    return n < glu::kCh / glu::kXc ? n : glu::kCh / glu::kXc;
}

// Shared state of the CTA's roles: a bounded wait that gives up when any
// role has given up.
struct Ctl {
    volatile int *abort;
    unsigned *flags;
    __device__ __forceinline__ bool wait(uint64_t *m, uint32_t parity) {
        uint32_t done = 0;
        for (uint32_t it = 0; it < glu::kSpinLimit && !done; ++it) {
            asm volatile(
                "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
                "selp.u32 %0, 1, 0, p;\n\t}\n"
                : "=r"(done)
                : "r"(umma::saddr(m)), "r"(parity)
                : "memory");
            if (!done && (it & 63) == 63 && *abort) return false;
        }
        if (!done) {
            *abort = 1;
            if (flags != nullptr) atomicOr(flags, S4_FLAG_TIMEOUT);
        }
        return done != 0;
    }
};

// a ring position: slot and the parity of its current use
struct Ring {
    int slot = 0;
    uint32_t phase = 0;
    __device__ __forceinline__ void next(int n) {
        if (++slot == n) {
            slot = 0;
            phase ^= 1u;
        }
    }
};

}  // namespace

// ---------------------------------------------------------------- layer norm
// One CTA: 64 consecutive time steps of one batch row, 4 per thread (16-byte
// accesses): thread (s, l) = (tid / 16, tid % 16) sums channels s, s + 16, ...
// at steps 4 l .. 4 l + 3, with 8 loads in flight; a warp reads two 256-byte
// channel rows per instruction. The sums are taken about x[b, 0, t] (shifted
// data: no cancellation for large means). The second pass re-reads the CTA's
// slab, which is still in L2. z may be x (in place): every element is read
// and then written by one thread.
__device__ __forceinline__ float4 f4sub(float4 a, float4 b) { return make_float4(a.x - b.x, a.y - b.y, a.z - b.z, a.w - b.w); }
__device__ __forceinline__ float4 f4add(float4 a, float4 b) { return make_float4(a.x + b.x, a.y + b.y, a.z + b.z, a.w + b.w); }
__device__ __forceinline__ float4 f4fma(float4 a, float4 b, float4 c) {
    return make_float4(fmaf(a.x, b.x, c.x), fmaf(a.y, b.y, c.y), fmaf(a.z, b.z, c.z), fmaf(a.w, b.w, c.w));
}

constexpr int kLnSteps = 64, kLnSlices = 16;

__global__ void __launch_bounds__(256) k_layernorm_channels(const float *x, const float *__restrict__ gamma,
                                                            const float *__restrict__ beta, float eps, int H,
                                                            int L, float *z) {
    __shared__ float4 s1[kLnSlices][kLnSteps / 4], s2[kLnSlices][kLnSteps / 4], mu_s[kLnSteps / 4],
        rs_s[kLnSteps / 4];
    const int tl = threadIdx.x % (kLnSteps / 4), hs = threadIdx.x / (kLnSteps / 4);
    const int t = blockIdx.x * kLnSteps + 4 * tl;
    const bool in = t < L;   // L is a multiple of 16: t < L implies t + 3 < L
    const size_t base = (size_t)blockIdx.y * H * L + t;
    const float4 zero = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    const float4 c = in ? *reinterpret_cast<const float4 *>(x + base) : zero;
    float4 a1 = zero, a2 = zero;
    if (in) {
#pragma unroll 8
        for (int h = hs; h < H; h += kLnSlices) {
            const float4 d = f4sub(*reinterpret_cast<const float4 *>(x + base + (size_t)h * L), c);
            a1 = f4add(a1, d);
            a2 = f4fma(d, d, a2);
        }
    }
    s1[hs][tl] = a1;
    s2[hs][tl] = a2;
    __syncthreads();
    if (hs == 0) {
        float4 S1 = zero, S2 = zero;
#pragma unroll
        for (int i = 0; i < kLnSlices; ++i) {
            S1 = f4add(S1, s1[i][tl]);
            S2 = f4add(S2, s2[i][tl]);
        }
        const float inv = 1.0f / (float)H;
        const float m[4] = {S1.x * inv, S1.y * inv, S1.z * inv, S1.w * inv};
        const float q[4] = {S2.x * inv, S2.y * inv, S2.z * inv, S2.w * inv};
        float r[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) r[i] = rsqrtf(fmaxf(q[i] - m[i] * m[i], 0.0f) + eps);
        mu_s[tl] = make_float4(c.x + m[0], c.y + m[1], c.z + m[2], c.w + m[3]);
        rs_s[tl] = make_float4(r[0], r[1], r[2], r[3]);
    }
    __syncthreads();
    if (!in) return;
    const float4 mu = mu_s[tl], rs = rs_s[tl];
#pragma unroll 8
    for (int h = hs; h < H; h += kLnSlices) {
        const size_t o = base + (size_t)h * L;
        const float4 v = *reinterpret_cast<const float4 *>(x + o);
        const float g = __ldg(gamma + h), bb = __ldg(beta + h);
        *reinterpret_cast<float4 *>(z + o) = make_float4((v.x - mu.x) * rs.x * g + bb, (v.y - mu.y) * rs.y * g + bb,
                                                          (v.z - mu.z) * rs.z * g + bb, (v.w - mu.w) * rs.w * g + bb);
    }
}

// H <= 16 NV: one pass. Thread (s, l) keeps channels s, s + 16, ... of its 4
// time steps in registers (all loads in flight at once); the mean and then
// the variance about it are two reductions over those registers, and z is
// written from them: x is read once.
template <int NV>
__global__ void __launch_bounds__(256, 2) k_layernorm_channels_reg(const float *x, const float *__restrict__ gamma,
                                                                const float *__restrict__ beta, float eps, int H,
                                                                int L, float *z) {
    __shared__ float4 sred[kLnSlices][kLnSteps / 4], sstat[kLnSteps / 4];
    const int tl = threadIdx.x % (kLnSteps / 4), hs = threadIdx.x / (kLnSteps / 4);
    const int t = blockIdx.x * kLnSteps + 4 * tl;
    const bool in = t < L;   // L is a multiple of 16: t < L implies t + 3 < L
    const size_t base = (size_t)blockIdx.y * H * L + t;
    const float4 zero = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    float4 v[NV];
#pragma unroll
    for (int i = 0; i < NV; ++i) {
        const int h = hs + kLnSlices * i;
        v[i] = (in && h < H) ? *reinterpret_cast<const float4 *>(x + base + (size_t)h * L) : zero;
    }
    const float inv = 1.0f / (float)H;
    float4 a = zero;
#pragma unroll
    for (int i = 0; i < NV; ++i) a = f4add(a, v[i]);
    sred[hs][tl] = a;
    __syncthreads();
    if (hs == 0) {
        float4 S = zero;
#pragma unroll
        for (int i = 0; i < kLnSlices; ++i) S = f4add(S, sred[i][tl]);
        sstat[tl] = make_float4(S.x * inv, S.y * inv, S.z * inv, S.w * inv);
    }
    __syncthreads();
    const float4 mu = sstat[tl];
    a = zero;
#pragma unroll
    for (int i = 0; i < NV; ++i)
        if (hs + kLnSlices * i < H) {
            const float4 d = f4sub(v[i], mu);
            a = f4fma(d, d, a);
        }
    __syncthreads();   // every thread has read sstat
    sred[hs][tl] = a;
    __syncthreads();
    if (hs == 0) {
        float4 S = zero;
#pragma unroll
        for (int i = 0; i < kLnSlices; ++i) S = f4add(S, sred[i][tl]);
        sstat[tl] = make_float4(rsqrtf(S.x * inv + eps), rsqrtf(S.y * inv + eps), rsqrtf(S.z * inv + eps),
                                rsqrtf(S.w * inv + eps));
    }
    __syncthreads();
    if (!in) return;
    const float4 rs = sstat[tl];
#pragma unroll
    for (int i = 0; i < NV; ++i) {
        const int h = hs + kLnSlices * i;
        if (h < H) {
            const float g = __ldg(gamma + h), bb = __ldg(beta + h);
            *reinterpret_cast<float4 *>(z + base + (size_t)h * L) =
                make_float4((v[i].x - mu.x) * rs.x * g + bb, (v[i].y - mu.y) * rs.y * g + bb,
                            (v[i].z - mu.z) * rs.z * g + bb, (v[i].w - mu.w) * rs.w * g + bb);
        }
    }
}

// ------------------------------------------------------- W -> operand images
// Image (c, nb): rows n of W' = W[128 nb + n/2] (n even) / W[H + 128 nb + n/2]
// (n odd), columns h = 32 c .. 32 c + 31, K-major, bf16 high part (first
// kWImg bytes) then low part; rows and columns past H are zero. Images are
// stored chunk-major, (c, nb) at ((c * nnb) + nb) * 2 kWImg. One thread
// writes 8 columns of one row.
__global__ void k_glu_prepare(const float *__restrict__ W, int H, unsigned char *__restrict__ img) {
    using namespace glu;
    const int nnb = glu_nnb(H);
    const long long total = (long long)glu_nkc(H) * nnb * kNr * (kKc / 8);
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= total) return;
    const int q = (int)(i % (kKc / 8));
    const int n = (int)((i / (kKc / 8)) % kNr);
    const long long cb = i / ((kKc / 8) * kNr);
    const int nb = (int)(cb % nnb), c = (int)(cb / nnb);
    const int o = nb * kCh + (n >> 1);
    const size_t wrow = (size_t)((n & 1) ? H + o : o) * H;
    float v[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const int h = c * kKc + 8 * q + j;
        v[j] = (o < H && h < H) ? W[wrow + h] : 0.0f;
    }
    uint4 hi, lo;
    split8(v, hi, lo);
    unsigned char *base = img + (size_t)cb * 2 * kWImg + kmajor_off(kNr, n, 8 * q);
    *reinterpret_cast<uint4 *>(base) = hi;
    *reinterpret_cast<uint4 *>(base + kWImg) = lo;
}

// ------------------------------------------- projection + GLU + residual
__global__ void __launch_bounds__(glu::kThreads, 1)
k_glu_projection_ws(const __grid_constant__ CUtensorMap tm_y, const __grid_constant__ CUtensorMap tm_x,
                    const float *__restrict__ bias, const unsigned char *__restrict__ wimg, int Bt, int H, int L,
                    int N, float *__restrict__ out, unsigned *flags) {
    using namespace glu;
    extern __shared__ __align__(1024) unsigned char sm[];
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + kOffBar);
    uint64_t *rawfull = bars, *rawempty = rawfull + kR;
    uint64_t *wfull = rawempty + kR, *yconv = wfull + kS, *opempty = yconv + kS;
    uint64_t *accfull = opempty + kS, *accempty = accfull + 2, *xfull = accempty + 2, *xempty = xfull + kX;
    uint32_t *tslot = reinterpret_cast<uint32_t *>(xempty + kX);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tslot + 1);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nnb = glu_nnb(H), nkc = glu_nkc(H), ntt = L / N;
    const long long ntiles = (long long)Bt * ntt * nnb;
    Ctl ctl{abort_flag, flags};

    if (tid == 0) {
        for (int i = 0; i < kR; ++i) {
            umma::mbar_init(&rawfull[i], 1);
            umma::mbar_init(&rawempty[i], 128);
        }
        for (int i = 0; i < kS; ++i) {
            umma::mbar_init(&wfull[i], 1);
            umma::mbar_init(&yconv[i], 128);
            umma::mbar_init(&opempty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            umma::mbar_init(&accfull[i], 1);
            umma::mbar_init(&accempty[i], kEpiThreads);
        }
        for (int i = 0; i < kX; ++i) {
            umma::mbar_init(&xfull[i], 1);
            umma::mbar_init(&xempty[i], kEpiThreads);
        }
        *abort_flag = 0;
        umma::fence_mbar_init();
    }
    if (warp == 5) umma::tmem_alloc(tslot, kTmemCols);
    umma::fence_before_sync();
    __syncthreads();
    umma::fence_after_sync();
    const uint32_t tmem = *tslot;

    if (warp == 0) {
        // ---------------- loader: raw y chunks (TMA) and W' image chunks (bulk)
        if (lane == 0) prefetch_tensormap(&tm_y);
        Ring rr, ss;
        // copies issued so far, counted per ring right after each issue: an
        // abort between the y copy and the W copy of one chunk leaves one
        // more y copy than W copies in flight, and the drain must see it
        int raw_issued = 0, w_issued = 0;
        bool ok = true;
        for (long long i = blockIdx.x; i < ntiles && ok; i += gridDim.x) {
            const Tile tl = tile_of(i, nnb, ntt, N);
            for (int c = 0; c < nkc; ++c) {
                if (!(ok = __all_sync(0xffffffffu, ctl.wait(&rawempty[rr.slot], rr.phase ^ 1u)))) break;
                if (lane == 0) {
                    arrive_expect_tx(&rawfull[rr.slot], (uint32_t)(N * kKc * 4));
                    tma_load_3d(sm + kOffRaw + rr.slot * kRawBytes, &tm_y, tl.t0, c * kKc, tl.b, &rawfull[rr.slot]);
                }
                ++raw_issued;
                rr.next(kR);
                if (!(ok = __all_sync(0xffffffffu, ctl.wait(&opempty[ss.slot], ss.phase ^ 1u)))) break;
                if (lane == 0) {
                    arrive_expect_tx(&wfull[ss.slot], 2 * kWImg);
                    bulk_load(sm + ss.slot * kStage + 2 * kYImg, wimg + ((size_t)c * nnb + tl.nb) * 2 * kWImg,
                              2 * kWImg, &wfull[ss.slot]);
                }
                __syncwarp();
                ++w_issued;
                ss.next(kS);
            }
        }
        if (!ok && lane == 0) {   // let the copies in flight land before the CTA exits
            for (int k = 1; k <= kR && k <= raw_issued; ++k) {
                const int u = raw_issued - k;
                umma::mbar_wait(&rawfull[u % kR], (uint32_t)((u / kR) & 1), kSpinLimit);
            }
            for (int k = 1; k <= kS && k <= w_issued; ++k) {
                const int u = w_issued - k;
                umma::mbar_wait(&wfull[u % kS], (uint32_t)((u / kS) & 1), kSpinLimit);
            }
        }
    } else if (warp <= 4) {
        // ---------------- converters: raw fp32 y chunk -> bf16 hi / lo operand image
        const int ct = tid - 32;   // time step within the tile (row of the operand)
        Ring rr, ss;
        bool ok = true;
        for (long long i = blockIdx.x; i < ntiles && ok; i += gridDim.x) {
            for (int c = 0; c < nkc; ++c) {
                if (!(ok = __all_sync(0xffffffffu, ctl.wait(&rawfull[rr.slot], rr.phase)))) break;
                if (!(ok = __all_sync(0xffffffffu, ctl.wait(&opempty[ss.slot], ss.phase ^ 1u)))) break;
                if (ct < N) {
                    const float *raw = reinterpret_cast<const float *>(sm + kOffRaw + rr.slot * kRawBytes);
                    unsigned char *img = sm + ss.slot * kStage;
#pragma unroll
                    for (int q = 0; q < kKc / 8; ++q) {
                        float v[8];
#pragma unroll
                        for (int j = 0; j < 8; ++j) v[j] = raw[(8 * q + j) * N + ct];
                        uint4 hi, lo;
                        split8(v, hi, lo);
                        const int off = kmajor_off(kTm, ct, 8 * q);
                        *reinterpret_cast<uint4 *>(img + off) = hi;
                        *reinterpret_cast<uint4 *>(img + kYImg + off) = lo;
                    }
                }
                umma::fence_proxy_async();   // the image, to the tensor cores
                arrive(&rawempty[rr.slot]);
                arrive(&yconv[ss.slot]);
                rr.next(kR);
                ss.next(kS);
            }
        }
    } else if (warp == 5) {
        // ---------------- MMA issue (one thread), accumulator a of tile k = k % 2
        const uint32_t id = umma::idesc(1, kTm, kNr);
        constexpr uint32_t y_lbo = (kTm / 8) * 128, w_lbo = (kNr / 8) * 128;
        Ring ss;
        uint32_t tl = 0;
        bool ok = true, any = false;
        for (long long i = blockIdx.x; i < ntiles && ok; i += gridDim.x, ++tl) {
            const int a = tl & 1;
            if (!(ok = __all_sync(0xffffffffu, ctl.wait(&accempty[a], ((tl >> 1) & 1u) ^ 1u)))) break;
            umma::fence_after_sync();
            for (int c = 0; c < nkc; ++c) {
                if (!(ok = __all_sync(0xffffffffu, ctl.wait(&wfull[ss.slot], ss.phase)))) break;
                if (!(ok = __all_sync(0xffffffffu, ctl.wait(&yconv[ss.slot], ss.phase)))) break;
                umma::fence_after_sync();
                if (lane == 0) {
                    const uint32_t yh = umma::saddr(sm + ss.slot * kStage), yl = yh + kYImg;
                    const uint32_t wh = yh + 2 * kYImg, wl = wh + kWImg;
                    const uint32_t As[3] = {yh, yh, yl}, Bs[3] = {wh, wl, wh};
#pragma unroll
                    for (int kk = 0; kk < kKc / 16; ++kk)
#pragma unroll
                        for (int pr = 0; pr < 3; ++pr)
                            umma::mma_bf16(tmem + (uint32_t)(a * kNr),
                                           umma::smem_desc(As[pr] + kk * 2 * y_lbo, y_lbo),
                                           umma::smem_desc(Bs[pr] + kk * 2 * w_lbo, w_lbo), id,
                                           c > 0 || kk > 0 || pr > 0);
                    umma::commit(&opempty[ss.slot]);
                }
                __syncwarp();
                any = true;
                ss.next(kS);
            }
            if (!ok) break;
            if (lane == 0) umma::commit(&accfull[a]);
            __syncwarp();
        }
        if (!ok && any && lane == 0) {   // let the issued MMAs finish before tensor memory is freed
            const int u = (ss.slot + kS - 1) % kS;
            umma::mbar_wait(&opempty[u], ss.slot == 0 ? ss.phase ^ 1u : ss.phase, kSpinLimit);
        }
    } else if (warp == 6) {
        // ---------------- x loader: residual chunks (tile, e) in order, into the x ring
        if (lane == 0) prefetch_tensormap(&tm_x);
        float *xs = reinterpret_cast<float *>(sm + kOffX);
        Ring xr;
        int issued = 0;
        bool ok = true;
        for (long long i = blockIdx.x; i < ntiles && ok; i += gridDim.x) {
            const Tile tc = tile_of(i, nnb, ntt, N);
            const int nx = x_chunks(H, tc.nb);
            for (int e = 0; e < nx; ++e) {
                if (!(ok = __all_sync(0xffffffffu, ctl.wait(&xempty[xr.slot], xr.phase ^ 1u)))) break;
                if (lane == 0) {
                    arrive_expect_tx(&xfull[xr.slot], (uint32_t)(N * kXc * 4));
                    tma_load_3d(xs + xr.slot * (kRawBytes / 4), &tm_x, tc.t0, tc.nb * kCh + e * kXc, tc.b,
                                &xfull[xr.slot]);
                }
                __syncwarp();
                ++issued;
                xr.next(kX);
            }
        }
        if (!ok && lane == 0)   // let the copies in flight land before the CTA exits
            for (int k = 1; k <= kX && k <= issued; ++k) {
                const int u = issued - k;
                umma::mbar_wait(&xfull[u % kX], (uint32_t)((u / kX) & 1), kSpinLimit);
            }
    } else {
        // ---------------- epilogue: warps 7..14; warp w reads tensor-memory lanes
        // 32 (w % 4) .. + 31 (time steps) and, of each 32-channel x chunk, the
        // 8-channel groups gh, gh + 1 (gh = 0 for warps 7-10, 2 for 11-14)
        const int q = warp & 3, t = 32 * q + lane;
        const int gh = warp < kEpiWarp0 + 4 ? 0 : 2;
        const float *xs = reinterpret_cast<const float *>(sm + kOffX);
        Ring xr;
        uint32_t tl = 0;
        bool ok = true;
        for (long long i = blockIdx.x; i < ntiles && ok; i += gridDim.x, ++tl) {
            const Tile tc = tile_of(i, nnb, ntt, N);
            const int a = tl & 1;
            if (!(ok = named_and(1, kEpiThreads, ctl.wait(&accfull[a], (tl >> 1) & 1u)))) break;
            umma::fence_after_sync();
            const int nx = x_chunks(H, tc.nb);
            const size_t row0 = ((size_t)tc.b * H) * L + tc.t0 + t;
            for (int e = 0; e < nx; ++e) {
                if (!(ok = named_and(1, kEpiThreads, ctl.wait(&xfull[xr.slot], xr.phase)))) break;
                const float *xc = xs + xr.slot * (kRawBytes / 4);
#pragma unroll
                for (int g = gh; g < gh + 2; ++g) {   // 16 columns = 8 channels
                    uint32_t v[16];
                    umma::ld_32x32b_x16(tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(a * kNr + e * 2 * kXc + 16 * g),
                                        v);
                    const int o0 = tc.nb * kCh + e * kXc + 8 * g;
                    float bv[8], bg[8];
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        bv[j] = o0 + j < H ? __ldg(bias + o0 + j) : 0.0f;
                        bg[j] = o0 + j < H ? __ldg(bias + H + o0 + j) : 0.0f;
                    }
                    if (t < N) {
#pragma unroll
                        for (int j = 0; j < 8; ++j) {
                            if (o0 + j < H) {
                                const float val = __uint_as_float(v[2 * j]) + bv[j];
                                const float gt = __uint_as_float(v[2 * j + 1]) + bg[j];
                                out[row0 + (size_t)(o0 + j) * L] = xc[(8 * g + j) * N + t] + val * sigmoidf_(gt);
                            }
                        }
                    }
                }
                arrive(&xempty[xr.slot]);   // this thread is done with the x slot
                xr.next(kX);
            }
            if (!ok) break;
            umma::fence_before_sync();
            arrive(&accempty[a]);
        }
    }
    umma::fence_before_sync();
    __syncthreads();
    umma::fence_after_sync();
    if (warp == 5) umma::tmem_dealloc(tmem, kTmemCols);
}

// ------------------------------------------------------------------ launchers
cudaError_t launch_layernorm_channels(const float *x, const float *gamma, const float *beta, float eps, int Bt,
                                      int H, int L, float *z, cudaStream_t st) {
    dim3 grid((L + kLnSteps - 1) / kLnSteps, Bt);
    if (H <= 4 * kLnSlices)
        k_layernorm_channels_reg<4><<<grid, 256, 0, st>>>(x, gamma, beta, eps, H, L, z);
    else if (H <= 16 * kLnSlices)
        k_layernorm_channels_reg<16><<<grid, 256, 0, st>>>(x, gamma, beta, eps, H, L, z);
    else
        k_layernorm_channels<<<grid, 256, 0, st>>>(x, gamma, beta, eps, H, L, z);
    return cudaGetLastError();
}

cudaError_t launch_glu_prepare(const float *W, int H, void *ws, cudaStream_t st) {
    const long long total = (long long)glu_nkc(H) * glu_nnb(H) * glu::kNr * (glu::kKc / 8);
    k_glu_prepare<<<(unsigned)((total + 255) / 256), 256, 0, st>>>(W, H, static_cast<unsigned char *>(ws));
    return cudaGetLastError();
}

namespace {
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;
int g_glu_sms[64];

// a [Bt, H, L] fp32 tensor as a 3-D TMA map with boxes [1][32][N]
cudaError_t tensor_map_bhl(CUtensorMap *m, const float *p, int Bt, int H, int L, int N) {
    std::call_once(g_encode_once, [] {
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", reinterpret_cast<void **>(&g_encode),
                                    cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            g_encode = nullptr;
    });
    if (g_encode == nullptr) return cudaErrorNotSupported;
    const cuuint64_t dims[3] = {(cuuint64_t)L, (cuuint64_t)H, (cuuint64_t)Bt};
    const cuuint64_t strides[2] = {(cuuint64_t)L * 4, (cuuint64_t)H * L * 4};
    const cuuint32_t box[3] = {(cuuint32_t)N, (cuuint32_t)glu::kKc, 1};
    const cuuint32_t es[3] = {1, 1, 1};
    const CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<float *>(p), dims, strides, box, es,
                                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                                CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}
}  // namespace

cudaError_t launch_glu_projection(const float *y, const float *x, const float *bias, const void *ws, int Bt, int H,
                                  int L, float *out, unsigned *flags, cudaStream_t st) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    int &sms = g_glu_sms[dev & 63];
    if (sms == 0) {
        e = cudaFuncSetAttribute(k_glu_projection_ws, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)glu::kSmem);
        if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return e;
    }
    const int N = L < glu::kTm ? L : glu::kTm;
    CUtensorMap my, mx;
    e = tensor_map_bhl(&my, y, Bt, H, L, N);
    if (e == cudaSuccess) e = tensor_map_bhl(&mx, x, Bt, H, L, N);
    if (e != cudaSuccess) return e;
    const long long tiles = (long long)Bt * (L / N) * glu_nnb(H);
    const int grid = tiles < sms ? (int)tiles : sms;
    k_glu_projection_ws<<<grid, glu::kThreads, glu::kSmem, st>>>(my, mx, bias, static_cast<const unsigned char *>(ws),
                                                                  Bt, H, L, N, out, flags);
    return cudaGetLastError();
}

}  // namespace s4
