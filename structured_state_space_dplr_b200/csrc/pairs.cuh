// pairs.cuh -- the two units of work of the forward pass for L <= 8192, as
// device functions of the kernels k_kgen and k_fftconv_pair:
//
//   kgen_channel : one channel's kernel K and the spectrum of the zero-padded
//                  K + D delta_0 ("The S4 kernel, from scratch", §4, §5):
//                  Cauchy/Woodbury generating function written straight into
//                  the inverse transform's digit-reversed input, length-L
//                  inverse transform -> K, whose last pass feeds the first
//                  pass of the length-2L forward transform;
//   conv_pair    : one row pair's causal convolution y = K * u + D u ([S4K]
//                  §5 fft_conv) with the spectrum above.
//
// Both run on one CTA of pair_threads<LG>() threads and use the same shared
// memory layout: two padded m-point buffers (the two halves of the 2L
// transform: rank 0 holds frequencies 2f, rank 1 frequencies 2f + 1), the
// middle-pass base twiddles, the first-pass tables a_j = W_2L^j, b_j = W_L^j,
// and an auxiliary area holding either the staged input rows (convolution)
// or the per-mode Cauchy constants (generation).
#pragma once
#include "cauchy.cuh"
#include "fft.cuh"

namespace s4 {

template <int LG>
__host__ __device__ constexpr int pair_threads() { return (1 << LG) / 16 < 32 ? 32 : (1 << LG) / 16; }
// CTAs per SM the pair kernels are built for: two up to L = 4096 (about
// 110 KB of shared memory each), one at L = 8192 (221 KB, 512 threads)
template <int LG>
__host__ __device__ constexpr int pair_min_blocks() { return LG <= 12 ? 2 : 1; }
template <int LG>
__host__ __device__ constexpr int pair_s0() { return (1 << LG) >> plan_lr(LG, 0); }
// float2 words before the auxiliary area (kept even: the area is 16-byte aligned)
template <int LG>
__host__ __device__ constexpr int pair_core_f2() {
    return (2 * padded(1 << LG) + plan_tw_size(LG) + 2 * pair_s0<LG>() + 1) / 2 * 2;
}
template <int LG>
__host__ __device__ constexpr size_t pair_smem_bytes(int Nh) {
    constexpr size_t cw = 2 * cauchy_mode_words<false>();   // float2 words of Cauchy constants per mode
    return sizeof(float2) * ((size_t)pair_core_f2<LG>() + ((size_t)(1 << LG) > cw * Nh ? (size_t)(1 << LG) : cw * Nh));
}

struct PairSmem {
    float2 *b0, *b1, *tws, *ta, *tb;
    float *stage;   // [2][L] input rows (convolution)
    float4 *sp;     // [3 Nh] Cauchy constants (generation, scalar form)
};

template <int LG>
__device__ __forceinline__ PairSmem pair_carve(float2 *sm) {
    constexpr int m = 1 << LG;
    PairSmem s;
    s.b0 = sm;
    s.b1 = sm + padded(m);
    s.tws = s.b1 + padded(m);
    s.ta = s.tws + plan_tw_size(LG);
    s.tb = s.ta + pair_s0<LG>();
    s.stage = reinterpret_cast<float *>(sm + pair_core_f2<LG>());
    s.sp = reinterpret_cast<float4 *>(sm + pair_core_f2<LG>());
    return s;
}

template <int LG>
__device__ __forceinline__ void pair_tables(const PairSmem &s) {
    constexpr int m = 1 << LG, T = pair_threads<LG>();
    for (int i = threadIdx.x; i < pair_s0<LG>(); i += T) {
        s.ta[i] = unit_root(i, 2 * m);
        s.tb[i] = unit_root(i, m);
    }
    build_middle_tables<LG>(s.tws, threadIdx.x, T);
}

// ------------------------------------------------------------ async copy --
__device__ __forceinline__ unsigned smem_u32(const void *p) { return (unsigned)__cvta_generic_to_shared(p); }
// 16-byte global -> shared copy (zero-filled when !valid; nothing is read then)
__device__ __forceinline__ void cp_async16(void *dst, const void *src, bool valid) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(smem_u32(dst)), "l"(src),
                 "r"(valid ? 16 : 0)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;\n" ::: "memory"); }

// Row pair pr = (channel h, rows 2 bp and 2 bp + 1) of u [Bt, H, L].
struct RowPair {
    int h, b0;
    bool has1;
};
__device__ __forceinline__ RowPair row_pair(long long pr, int Bt) {
    const int nbp = (Bt + 1) / 2;
    RowPair r;
    r.h = (int)(pr / nbp);
    r.b0 = 2 * (int)(pr % nbp);
    r.has1 = r.b0 + 1 < Bt;
    return r;
}

// Both rows of pair pr into the stage (cp.async, then committed).
template <int LG>
__device__ __forceinline__ void pair_stage_rows(const PairSmem &s, const float *__restrict__ u, int Bt, int H,
                                                long long pr) {
    constexpr int L = 1 << LG, T = pair_threads<LG>();
    const RowPair r = row_pair(pr, Bt);
    const float *u0 = u + ((size_t)r.b0 * H + r.h) * L;
    const float *u1 = r.has1 ? u0 + (size_t)H * L : u0;
    for (int i = threadIdx.x; i < L / 2; i += T) {   // 16-byte chunks, L/4 per row
        const int row = i >= L / 4, k = (i - row * (L / 4)) * 4;
        cp_async16(s.stage + row * L + k, (row ? u1 : u0) + k, !row || r.has1);
    }
    cp_async_commit();
}

// ------------------------------------------------------ both halves, pass 0 --
// First forward pass of group j of both halves of the zero-padded length-2m
// transform: half 0 transforms v0, half 1 transforms v1 after the twist
// W_2m^-k, whose in-group share W_2R0^-p is a constant rotation and whose
// remainder a_j b_j^q is applied with the group twiddles b_j^q (v0, v1: the
// group's inputs, point j + p S0). SCALE also multiplies every output of the
// group by f (a twist constant over the group).
template <int LG, bool SCALE>
__device__ __forceinline__ void first_pass_halves2(const PairSmem &s, const float2 (&v0)[1 << plan_lr(LG, 0)],
                                                   const float2 (&v1)[1 << plan_lr(LG, 0)], int j, float2 f) {
    constexpr int R0 = 1 << plan_lr(LG, 0), S0 = (1 << LG) / R0;
    float2 x[R0], z[R0];
    static_for<0, R0>([&](auto p) {
        x[p] = v0[p];
        z[p] = rot<decltype(p)::value, 2 * R0, -1>(v1[p]);
    });
    dft<R0, -1>(x);
    dft<R0, -1>(z);
    const float2 a = s.ta[j], b = s.tb[j];
    const int o = pidx(j);
    if constexpr (SCALE) {
        float2 w = f, u = cmul(f, a);
        s.b0[o] = cmul(x[0], w);
        s.b1[o] = cmul(z[0], u);
        static_for<1, R0>([&](auto q) {
            w = cmul(w, b);
            u = cmul(u, b);
            s.b0[o + poff<decltype(q)::value * S0>()] = cmul(x[q], w);
            s.b1[o + poff<decltype(q)::value * S0>()] = cmul(z[q], u);
        });
    } else {
        float2 w = b, u = a;
        s.b0[o] = x[0];
        s.b1[o] = cmul(z[0], a);
        static_for<1, R0>([&](auto q) {
            u = cmul(u, b);
            s.b0[o + poff<decltype(q)::value * S0>()] = cmul(x[q], w);
            s.b1[o + poff<decltype(q)::value * S0>()] = cmul(z[q], u);
            w = cmul(w, b);
        });
    }
}
// both halves from the same m nonzero inputs (the zero-padded length-2m transform)
template <int LG>
__device__ __forceinline__ void first_pass_halves(const PairSmem &s, const float2 (&v)[1 << plan_lr(LG, 0)],
                                                  int j) {
    first_pass_halves2<LG, false>(s, v, v, j, make_float2(1.0f, 0.0f));
}

// After the first pass of both halves (stored, all threads synced): forward
// passes 1 .. P-1, then (spectrum + D) * scale in spec4_index order, half 0
// to o0 and half 1 to o1. Adding D to every frequency adds D delta_0 to K.
template <int LG>
__device__ __forceinline__ void spectrum_tail2(const PairSmem &s, float Dh, float scale, float4 *__restrict__ o0,
                                               float4 *__restrict__ o1) {
    constexpr int m = 1 << LG, T = pair_threads<LG>();
    constexpr int R = 1 << plan_lr(LG, plan_P(LG) - 1);
    forward_middle_x2<LG, T>(s.b0, s.b1, s.tws);
    for (int g = threadIdx.x; g < m / R; g += T) {
        const int base = g * R, o = pidx(base);
        float2 x[R], z[R];
        load_contig<R>(s.b0 + o, x);
        load_contig<R>(s.b1 + o, z);
        dft<R, -1>(x);
        dft<R, -1>(z);
        static_for<0, R / 2>([&](auto i) {
            o0[spec4_index<LG>(base, i)] = make_float4((x[2 * i].x + Dh) * scale, x[2 * i].y * scale,
                                                       (x[2 * i + 1].x + Dh) * scale, x[2 * i + 1].y * scale);
            o1[spec4_index<LG>(base, i)] = make_float4((z[2 * i].x + Dh) * scale, z[2 * i].y * scale,
                                                       (z[2 * i + 1].x + Dh) * scale, z[2 * i + 1].y * scale);
        });
    }
}
// the length-2m spectrum of one channel: rank 0 then rank 1, scaled by 1/2m
template <int LG>
__device__ __forceinline__ void spectrum_tail(const PairSmem &s, float Dh, float2 *__restrict__ spec_h) {
    constexpr int m = 1 << LG;
    float4 *o0 = reinterpret_cast<float4 *>(spec_h);
    spectrum_tail2<LG>(s, Dh, 1.0f / (float)(2 * m), o0, o0 + m / 2);
}

// The same spectrum from K[h, :] in global memory (tables built, all threads
// synced on entry).
template <int LG>
__device__ __forceinline__ void kspec_channel(const PairSmem &s, const float *__restrict__ Kh, float Dh,
                                              float2 *__restrict__ spec_h) {
    constexpr int m = 1 << LG, T = pair_threads<LG>();
    constexpr int R0 = 1 << plan_lr(LG, 0), S0 = m / R0;
    for (int j = threadIdx.x; j < S0; j += T) {
        float2 v[R0];
        static_for<0, R0>([&](auto p) { v[p] = make_float2(__ldg(Kh + j + p * S0), 0.0f); });
        first_pass_halves<LG>(s, v, j);
    }
    __syncthreads();
    spectrum_tail<LG>(s, Dh, spec_h);
}

// Last inverse pass of both halves (all threads synced on entry): output
// point t < m of the length-2m inverse is half 0's value plus half 1's, the
// latter twisted back by W_2m^t (in-group share W_2R0^p); out(p, t, sum,
// diff) receives that sum and the difference (half 0 minus half 1), with p
// (t = j + p S0) as a compile-time constant.
template <int LG, class Out>
__device__ __forceinline__ void last_pass_halves_sum(const PairSmem &s, Out &&out) {
    constexpr int m = 1 << LG, T = pair_threads<LG>();
    constexpr int R0 = 1 << plan_lr(LG, 0), S0 = m / R0;
    for (int j = threadIdx.x; j < S0; j += T) {
        float2 x[R0], z[R0];
        const int o = pidx(j);
        const float2 a = s.ta[j], b = s.tb[j];
        float2 w = b, v = a;
        x[0] = s.b0[o];
        z[0] = cmulc(s.b1[o], a);
        static_for<1, R0>([&](auto q) {
            v = cmul(v, b);
            x[q] = cmulc(s.b0[o + poff<decltype(q)::value * S0>()], w);
            z[q] = cmulc(s.b1[o + poff<decltype(q)::value * S0>()], v);
            w = cmul(w, b);
        });
        dft<R0, +1>(x);
        dft<R0, +1>(z);
        static_for<0, R0>([&](auto p) {
            const float2 rz = rot<decltype(p)::value, 2 * R0, +1>(z[p]);
            out(p, j + p * S0, cadd(x[p], rz), csub(x[p], rz));
        });
    }
}

// ------------------------------------------------------------ convolution --
// Convolution of the staged row pair (stage ready, all threads synced) with
// the spectrum spec_h (layout of spec4_index, rank 0 then rank 1). After the
// first pass, after_first() runs (the stage is free then). CONJ multiplies
// by the conjugate spectrum instead: the adjoint, a correlation
// y[s] = sum_{t >= s} K[t - s] u[t] + D u[s] (K and D are real).
template <int LG, bool CONJ, class AfterFirst>
__device__ __forceinline__ void conv_pair(const PairSmem &s, const float2 *__restrict__ spec_h, float *y0,
                                          float *y1, bool has1, AfterFirst &&after_first) {
    constexpr int m = 1 << LG, L = m, T = pair_threads<LG>();
    constexpr int R0 = 1 << plan_lr(LG, 0), S0 = m / R0;
    float2 *b0 = s.b0, *b1 = s.b1;
    const float *stage = s.stage;
    // ---- first forward pass, both halves: input u0 + i u1
    for (int j = threadIdx.x; j < S0; j += T) {
        float2 v[R0];
        static_for<0, R0>([&](auto p) {
            const int k = j + p * S0;
            v[p] = make_float2(stage[k], stage[L + k]);
        });
        first_pass_halves<LG>(s, v, j);
    }
    __syncthreads();
    after_first();
    const float4 *s0 = reinterpret_cast<const float4 *>(spec_h);
    const float4 *s1 = s0 + m / 2;
    constexpr int RL = 1 << plan_lr(LG, plan_P(LG) - 1);
    struct SpecWords { float4 k0[RL / 2], k1[RL / 2]; };
    auto fetch = [&](int base) {
        SpecWords w;
        static_for<0, RL / 2>([&](auto i) {
            w.k0[i] = __ldg(s0 + spec4_index<LG>(base, i));
            w.k1[i] = __ldg(s1 + spec4_index<LG>(base, i));
        });
        return w;
    };
    auto product = [&](const SpecWords &w, auto &x, auto &z) {
        auto mul = [](float2 a, float x0, float x1) {
            if constexpr (CONJ) return cmulc(a, make_float2(x0, x1)); else return cmul(a, make_float2(x0, x1));
        };
        static_for<0, RL / 2>([&](auto i) {
            x[2 * i] = mul(x[2 * i], w.k0[i].x, w.k0[i].y);
            x[2 * i + 1] = mul(x[2 * i + 1], w.k0[i].z, w.k0[i].w);
            z[2 * i] = mul(z[2 * i], w.k1[i].x, w.k1[i].y);
            z[2 * i + 1] = mul(z[2 * i + 1], w.k1[i].z, w.k1[i].w);
        });
    };
    if constexpr (warp_local_middle<LG, T, 2>()) {   // barriers between the middle passes per warp
        pass_x2<LG, 1, -1, false, T>(b0, b1, s.tws);
        __syncwarp();
        if constexpr (plan_lr(LG, 1) == 5) fused_blocks<LG, 2, CONJ>(b0, b1, s0, s1);
        else fused_middle_x2<LG, T>(b0, b1, fetch, product);
        __syncwarp();
        pass_x2<LG, 1, +1, true, T>(b0, b1, s.tws);
        __syncthreads();
    } else {
        forward_middle_x2<LG, T>(b0, b1, s.tws);
        fused_middle_x2<LG, T>(b0, b1, fetch, product);
        __syncthreads();
        inverse_middle_x2<LG, T>(b0, b1, s.tws);
    }
    // ---- last inverse pass of both halves + their sum, straight to y
    last_pass_halves_sum<LG>(s, [&](auto, int t, float2 r, float2) {
        y0[t] = r.x;
        if (has1) y1[t] = r.y;
    });
}

// ------------------------------------------------------------- generation --
// Channel h: K[h, :] and spec_h (2L complex, spec4_index layout, scaled by
// 1/2L, with D added). Tables built, all threads synced on entry.
template <int LG>
__device__ __forceinline__ void kgen_channel(const PairSmem &s, const float2 *__restrict__ Lambda,
                                             const float2 *__restrict__ P, const float2 *__restrict__ Q,
                                             const float2 *__restrict__ B, const float2 *__restrict__ Cc,
                                             const float *__restrict__ log_dt, const float *__restrict__ D,
                                             int Nh, int h, float *__restrict__ K, float2 *__restrict__ spec_h,
                                             unsigned *__restrict__ flags) {
    constexpr int m = 1 << LG, L = m, T = pair_threads<LG>();
    constexpr int R0 = 1 << plan_lr(LG, 0), S0 = m / R0, NP = plan_P(LG);
    constexpr int F = 4;   // frequencies per thread per round
    float2 *X = s.b0;   // the length-L inverse transform
    float4 *sp = s.sp;
    cauchy_stage_modes<false>(Lambda, P, Q, B, Cc, h, Nh, sp, flags, threadIdx.x, T);
    __syncthreads();

    // ---- A: generating function -> X at digit-reversed positions (with mirror)
    // Threads walk the positions that hold frequencies j < L/2 rather than
    // the frequencies themselves: the top digit of j is the low digit of its
    // position p (the radix RL of the last pass), so j < L/2 exactly when
    // p mod RL < RL/2. Slot q goes to p = (q mod RL/2) + RL b', with the
    // blocks b' of consecutive slots interleaved so that the two 8-lane
    // halves of a half-warp store 4 blocks (8 bank slots) apart: the stores
    // of a warp hit distinct banks (their mirrors at most two ways), where
    // consecutive frequencies would land 256 points apart, all in one bank.
    const float ldt = __ldg(log_dt + h);
    const float inv_dt = expf(-ldt);
    constexpr int RL = 1 << plan_lr(LG, NP - 1), HB = RL / 2;
    constexpr bool SPREAD = HB == 8 && (L / RL) % 8 == 0;
    auto slot_pos = [](int q) {
        const int b = q / HB;
        const int bb = SPREAD ? ((b & ~7) | ((b & 1) << 2) | ((b >> 1) & 3)) : b;
        return q % HB + RL * bb;
    };
    bool bad = false;
    for (int f0 = 0; f0 < L / 2; f0 += T * F) {
        int q[F], pos[F], jj[F];
#pragma unroll
        for (int f = 0; f < F; ++f) {
            q[f] = f0 + f * T + threadIdx.x;
            pos[f] = slot_pos(q[f] < L / 2 ? q[f] : 0);
            jj[f] = digrev<LG>(pos[f]);   // < L/2
        }
        float2 kh[F];
        cauchy_eval<F, false>(sp, Nh, jj, L, inv_dt, kh);
#pragma unroll
        for (int f = 0; f < F; ++f) {
            if (q[f] < L / 2) {
                bad |= !(isfinite(kh[f].x) && isfinite(kh[f].y));
                if (jj[f] == 0) {
                    X[pidx(0)] = make_float2(kh[f].x, 0.0f);
                } else {
                    X[pidx(pos[f])] = kh[f];
                    X[pidx(digrev_inv<LG>(L - jj[f]))] = cconj(kh[f]);
                }
            }
        }
    }
    if (threadIdx.x == 0) {
        const float nyq = cauchy_nyquist<false>(sp, Nh, expf(ldt), L);
        bad |= !isfinite(nyq);
        X[pidx(digrev_inv<LG>(L / 2))] = make_float2(nyq, 0.0f);
    }
    if (flags != nullptr && __any_sync(0xffffffffu, bad) && (threadIdx.x & 31) == 0)
        atomicOr(flags, S4_FLAG_NONFINITE);
    __syncthreads();

    // ---- B: inverse transform, passes P-1 .. 1
    dit_pass<LG, NP - 1, +1, T>(X, s.tws);
    __syncthreads();
    inverse_middle<LG, T>(X, s.tws);

    // ---- B/C: last inverse pass -> K (stored); its registers start the
    // first forward pass of both halves (same group, same positions)
    float *Kh = K + (size_t)h * L;
    for (int j = threadIdx.x; j < S0; j += T) {
        const int o = pidx(j);
        const float2 b = s.tb[j];
        float2 x[R0];
        float2 w = b;
        x[0] = X[o];
        static_for<1, R0>([&](auto q) {
            x[q] = cmulc(X[o + poff<decltype(q)::value * S0>()], w);
            w = cmul(w, b);
        });
        dft<R0, +1>(x);
        static_for<0, R0>([&](auto p) {
            const float k = x[p].x;   // K is real: the imaginary part is rounding
            Kh[j + p * S0] = k;
            x[p] = make_float2(k, 0.0f);
        });
        first_pass_halves<LG>(s, x, j);
    }
    __syncthreads();

    // ---- C: forward passes 1 .. P-1 -> (spectrum + D) / 2L
    spectrum_tail<LG>(s, D != nullptr ? __ldg(D + h) : 0.0f, spec_h);
}

}  // namespace s4
