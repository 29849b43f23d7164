// Channel scan of the Mamba-1 configuration ("When a Diagonal State Is Not
// Enough", sungsoo.github.io, Part 01 "Definition", with the Mamba-1 recovery of
// Part 04; "State Space Models", robocikowo.com, glossary item 2): every channel
// is its own head with head dim 1 and N = 8 or 16 real state rows with their
// own decays, dt per (token, channel), B_t and C_t shared by the channels of a
// group, bf16 I/O, fp32 state; optional two-endpoint writes.
//
// The work is a sequential recurrence per channel whose cost is one exp per
// (token, channel, state row): the special-function unit (MUFU) bounds it.
// A thread keeps 4 state rows of one channel in registers (S = N / 4 threads
// per channel, their readouts summed with shuffles) and walks the sequence;
// 64 channels form a CTA, which
// stages 16 tokens of dt, lambda, x (and dy), B_t and C_t in shared memory with
// cp.async, double-buffered, so that the loads of the next tile overlap the
// recurrence of this one.  Pre-state form K_t = A_t K_{t-1} + sigma_t B_t x_t,
// y_t = C_t . K_t + (D - beta_{t+1} C_t . B_t) x_t.
//
// Forward (k_m1_fwd): the recurrence; a training forward also keeps K at the
// start of every 16-token tile for the backward.
// Backward (k_m1_bwd): tiles in reverse; per tile the states are recomputed
// from the kept K into shared memory, then the adjoint G = dL/dK walks the tile
// backwards with every gradient taken per step, exactly:
//   dK_t += C_t dy_t;  dsigma_t = x_t <B_t, G>;  dx_t = (D - beta_{t+1} C.B) dy_t + sigma_t <B_t, G>
//   drho_{t,n} = G_n A_{t,n} K_{t-1,n}  (rho = dt a: the log-decay of step t)
//   dB_t += sigma_t x_t G - beta_{t+1} x_t dy_t C_t,  dC_t += dy_t K_t - beta_{t+1} x_t dy_t B_t
//   G <- A_t G
// dB and dC are summed over the CTA's channels with shuffles in a fixed order and
// leave as per-CTA partials; k_m1_bc_sum adds the partials of a group in order.
#include <cuda_bf16.h>

#include "common.cuh"

namespace ssm {
namespace m1 {

constexpr int CPB = 64;   // channels per CTA
constexpr int TT = 16;    // tokens per staged tile
constexpr int NSL = 4;    // state rows per thread

__device__ __forceinline__ float bfu(unsigned short v) { return __uint_as_float((uint32_t)v << 16); }

__device__ __forceinline__ void cp_async16(void *dst, const void *src, bool ok) {
    const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(dst));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(d), "l"(src),
                 "r"(ok ? 16 : 0)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int K>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;\n" ::"n"(K) : "memory");
}

// one staged tile: dt / lambda of TT + 1 tokens (beta_{t+1}), x / dy of TT tokens,
// B_t / C_t of TT tokens (N <= 16), all raw bf16
struct Tile {
    unsigned short dt[TT + 1][CPB], lam[TT + 1][CPB], x[TT][CPB], dy[TT][CPB];
    unsigned short B[TT][16], C[TT][16];
};

// Issue the cp.async copies of the tile starting at token t0 (rows past L are
// zero-filled; `src_ok` false rows read a valid dummy address).
__device__ __forceinline__ void stage(const Params &p, Tile &tl, int b, int hb, int g, int t0,
                                      bool with_dy) {
    const int nthr = blockDim.x;
    const unsigned short *dt = reinterpret_cast<const unsigned short *>(p.dt);
    const unsigned short *lam = reinterpret_cast<const unsigned short *>(p.lam);
    const unsigned short *x = reinterpret_cast<const unsigned short *>(p.x);
    const unsigned short *dy = reinterpret_cast<const unsigned short *>(p.dy);
    const unsigned short *Bm = reinterpret_cast<const unsigned short *>(p.Bm);
    const unsigned short *Cm = reinterpret_cast<const unsigned short *>(p.Cm);
    for (int i = threadIdx.x; i < (TT + 1) * 8; i += nthr) {
        const int r = i >> 3, c8 = 8 * (i & 7), t = t0 + r;
        const bool ok = t < p.L;
        cp_async16(&tl.dt[r][c8], ok ? dt + ix_dt(p, b, t, hb + c8) : dt, ok);
        if (p.two_ep) cp_async16(&tl.lam[r][c8], ok ? lam + ix_lam(p, b, t, hb + c8) : lam, ok);
    }
    for (int i = threadIdx.x; i < TT * 8; i += nthr) {
        const int r = i >> 3, c8 = 8 * (i & 7), t = t0 + r;
        const bool ok = t < p.L;
        cp_async16(&tl.x[r][c8], ok ? x + ix_x(p, b, t, hb + c8, 0, 0) : x, ok);
        if (with_dy) cp_async16(&tl.dy[r][c8], ok ? dy + ix_y(p, b, t, hb + c8, 0, 0) : dy, ok);
    }
    const int nb = p.N / 8;
    for (int i = threadIdx.x; i < TT * nb; i += nthr) {
        const int r = i / nb, k8 = 8 * (i % nb), t = t0 + r;
        const bool ok = t < p.L;
        cp_async16(&tl.B[r][k8], ok ? Bm + ix_B(p, b, t, g, 0, k8) : Bm, ok);
        cp_async16(&tl.C[r][k8], ok ? Cm + ix_C(p, b, t, g, 0, k8) : Cm, ok);
    }
    cp_async_commit();
}

// 4 consecutive bf16 (8-byte aligned) as floats
__device__ __forceinline__ void ld4(const unsigned short *src, float (&v)[NSL]) {
    const uint2 w = *reinterpret_cast<const uint2 *>(src);
    v[0] = __uint_as_float(w.x << 16);
    v[1] = __uint_as_float(w.x & 0xffff0000u);
    v[2] = __uint_as_float(w.y << 16);
    v[3] = __uint_as_float(w.y & 0xffff0000u);
}
// sum over the S lanes of a channel (consecutive lanes)
template <int S>
__device__ __forceinline__ float lane_sum(float v) {
#pragma unroll
    for (int m = 1; m < S; m <<= 1) v += __shfl_xor_sync(0xffffffffu, v, m);
    return v;
}

__device__ __forceinline__ float ex2f(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// decay rates (times log2 e) of this thread's state rows
__device__ __forceinline__ void rates(const Params &p, int h, int half, float (&a)[NSL],
                                      float (&a2)[NSL]) {
#pragma unroll
    for (int i = 0; i < NSL; ++i) {
        const int n = NSL * half + i;
        a[i] = -expf(__ldg(p.A_log + h * p.ndec + (p.per_coord ? n : 0)));
        a2[i] = a[i] * 1.4426950408889634f;
    }
}

}  // namespace m1

// ============================================================================
template <int S>
__global__ void __launch_bounds__(64 * S, 2) k_m1_fwd(Params p, float *kept) {
    using namespace m1;
    __shared__ __align__(16) Tile tiles[2];
    __shared__ float s_cb[2][TT];
    __shared__ __align__(16) unsigned short s_y[TT][CPB];
    const int tid = threadIdx.x, ch = tid / S, half = tid % S;
    const int hb = blockIdx.x * CPB, h = hb + ch, b = blockIdx.y;
    const int g = hb / p.hpg;
    const int L = p.L, ntile = (L + TT - 1) / TT;
    float a[NSL], a2[NSL], K[NSL];
    rates(p, h, half, a, a2);
    const float D = (p.R == p.O && p.D) ? __ldg(p.D + h) : 0.f;
    {   // K_{-1} = h0 + beta_0 w0
        float beta0 = 0.f;
        if (p.two_ep && L > 0)
            beta0 = (1.f - ld_io(p.lam, ix_lam(p, b, 0, h), 1)) * ld_io(p.dt, ix_dt(p, b, 0, h), 1);
#pragma unroll
        for (int i = 0; i < NSL; ++i) {
            const long long ii = ix_st(p, b, h, NSL * half + i, 0);
            float v = p.h0 ? p.h0[ii] : 0.f;
            if (p.w0) v = fmaf(beta0, p.w0[ii], v);
            K[i] = v;
        }
    }
    if (ntile > 0) stage(p, tiles[0], b, hb, g, 0, false);
    for (int k = 0; k < ntile; ++k) {
        const int buf = k & 1, t0 = k * TT;
        Tile &tl = tiles[buf];
        if (k + 1 < ntile) {
            stage(p, tiles[buf ^ 1], b, hb, g, t0 + TT, false);
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncthreads();
        if (tid < TT) {   // C_t . B_t of the tile's tokens
            float s = 0.f;
            for (int n = 0; n < p.N; ++n) s = fmaf(bfu(tl.C[tid][n]), bfu(tl.B[tid][n]), s);
            s_cb[buf][tid] = s;
        }
        if (kept) {   // the state entering this tile, for the backward
            float *dst = kept + (((long long)b * p.H + h) * ntile + k) * p.N + NSL * half;
            *reinterpret_cast<float4 *>(dst) = make_float4(K[0], K[1], K[2], K[3]);
        }
        __syncthreads();
#pragma unroll 4
        for (int j = 0; j < TT; ++j) {
            const int t = t0 + j;
            const float dt = bfu(tl.dt[j][ch]), x = bfu(tl.x[j][ch]);
            float lam = 1.f, bn = 0.f;
            if (p.two_ep) {
                lam = bfu(tl.lam[j][ch]);
                if (t + 1 < L) bn = (1.f - bfu(tl.lam[j + 1][ch])) * bfu(tl.dt[j + 1][ch]);
            }
            const float w = fmaf(lam, dt, bn) * x;
            float Bv[NSL], Cv[NSL];
            ld4(&tl.B[j][NSL * half], Bv);
            ld4(&tl.C[j][NSL * half], Cv);
            float yp = 0.f;
#pragma unroll
            for (int i = 0; i < NSL; ++i) {
                K[i] = fmaf(ex2f(a2[i] * dt), K[i], w * Bv[i]);
                yp = fmaf(Cv[i], K[i], yp);
            }
            yp = lane_sum<S>(yp);
            if (half == 0)
                s_y[j][ch] = __bfloat16_as_ushort(
                    __float2bfloat16_rn(fmaf(fmaf(-bn, s_cb[buf][j], D), x, yp)));
        }
        __syncthreads();
        if (p.y) {   // the tile's y rows, 16 bytes per thread
            for (int i = tid; i < TT * 8; i += 64 * S) {
                const int r = i >> 3, c8 = 8 * (i & 7);
                if (t0 + r < L)
                    *reinterpret_cast<uint4 *>(reinterpret_cast<unsigned short *>(p.y) +
                                               ix_y(p, b, t0 + r, hb + c8, 0, 0)) =
                        *reinterpret_cast<const uint4 *>(&s_y[r][c8]);
            }
        }
    }
    // final state (beta_L = 0, so K_{L-1} = H_{L-1}) and the last write B_{L-1} x_{L-1}
    if (L > 0) {
        const float xl = ld_io(p.x, ix_x(p, b, L - 1, h, 0, 0), 1);
#pragma unroll
        for (int i = 0; i < NSL; ++i) {
            const int n = NSL * half + i;
            const long long ii = ix_st(p, b, h, n, 0);
            if (p.hT) p.hT[ii] = K[i];
            if (p.wT) p.wT[ii] = ld_io(p.Bm, ix_B(p, b, L - 1, g, 0, n), 1) * xl;
        }
    }
}

// ============================================================================
// Sum of 2 NSL = 8 values over the 32 / S lanes of a warp that hold the same
// rows of different channels (lane = S * channel + sub): butterfly
// reduce-scatter over lane bits 16 .. S in a fixed order.  Afterwards lane l
// holds, in v[0], the total of value (l >> 2) & 7 of its `sub` (for S = 2 the
// last level adds lane pairs that already hold the same value index, so both
// lanes of a pair end with the same total).
template <int S>
__device__ __forceinline__ void chan_reduce8(float (&v)[2 * m1::NSL], int lane) {
    int cur = 2 * m1::NSL;
#pragma unroll
    for (int m = 16; m >= S; m >>= 1) {
        if (cur > 1) {
            const bool up = (lane & m) != 0;
            const int hl = cur / 2;
#pragma unroll
            for (int i = 0; i < m1::NSL; ++i) {
                if (i < hl) {
                    const float send = up ? v[i] : v[i + hl];
                    const float keep = up ? v[i + hl] : v[i];
                    v[i] = keep + __shfl_xor_sync(0xffffffffu, send, m);
                }
            }
            cur = hl;
        } else {
            v[0] += __shfl_xor_sync(0xffffffffu, v[0], m);
        }
    }
}

template <int S>
__global__ void __launch_bounds__(64 * S, 2) k_m1_bwd(Params p, const float *kept, float *bc_part,
                                                      float *par_part) {
    using namespace m1;
    constexpr int NT = 64 * S;
    constexpr int NW = NT / 32;
    extern __shared__ __align__(16) unsigned char m1_smem[];
    Tile *tiles = reinterpret_cast<Tile *>(m1_smem);
    float *Ks = reinterpret_cast<float *>(m1_smem + 2 * sizeof(Tile));   // [TT + 1][NSL][NT]
    float *red = Ks + (TT + 1) * NSL * NT;                               // [NW][TT][32]
    float *s_cb = red + NW * TT * 32;                                    // [TT]
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int ch = tid / S, half = tid % S;
    const int hb = blockIdx.x * CPB, h = hb + ch, b = blockIdx.y;
    const int g = hb / p.hpg;
    const int L = p.L, ntile = (L + TT - 1) / TT;
    const int nblk = p.hpg / CPB, blk = (hb % p.hpg) / CPB;   // CTAs of the group, this one
    float a[NSL], a2[NSL], G[NSL], dA[NSL];
    rates(p, h, half, a, a2);
    const float D = (p.R == p.O && p.D) ? __ldg(p.D + h) : 0.f;
#pragma unroll
    for (int i = 0; i < NSL; ++i) G[i] = dA[i] = 0.f;
    float dD = 0.f;
    // token t + 1 waits for dbeta_{t+1}, which step t produces
    float pend_base = 0.f, pend_lam = 1.f, pend_dt = 0.f, pend_dgam = 0.f;
    int pend_t = -1;
    auto finish = [&](float dbeta) {
        if (pend_t < 0 || half != 0) return;
        const float ddt = fmaf(1.f - pend_lam, dbeta, pend_base);
        st_io(p.ddt, ix_dt(p, b, pend_t, h), ddt, 1);
        if (p.two_ep && p.dlam) st_io(p.dlam, ix_lam(p, b, pend_t, h), pend_dt * (pend_dgam - dbeta), 1);
    };
    if (ntile > 0) stage(p, tiles[(ntile - 1) & 1], b, hb, g, (ntile - 1) * TT, true);
    for (int k = ntile - 1; k >= 0; --k) {
        const int buf = k & 1, t0 = k * TT;
        Tile &tl = tiles[buf];
        if (k > 0) {
            stage(p, tiles[buf ^ 1], b, hb, g, t0 - TT, true);
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncthreads();
        if (tid < TT) {
            float s = 0.f;
            for (int n = 0; n < p.N; ++n) s = fmaf(bfu(tl.C[tid][n]), bfu(tl.B[tid][n]), s);
            s_cb[tid] = s;
        }
        // ---- the tile's states from the kept entering state ------------------------
        {
            const float *src = kept + (((long long)b * p.H + h) * ntile + k) * p.N + NSL * half;
            const float4 k0 = __ldg(reinterpret_cast<const float4 *>(src));
            float K[NSL] = {k0.x, k0.y, k0.z, k0.w};
#pragma unroll
            for (int i = 0; i < NSL; ++i) Ks[i * NT + tid] = K[i];
#pragma unroll 4
            for (int j = 0; j < TT; ++j) {
                const int t = t0 + j;
                const float dt = bfu(tl.dt[j][ch]), x = bfu(tl.x[j][ch]);
                float lam = 1.f, bn = 0.f;
                if (p.two_ep) {
                    lam = bfu(tl.lam[j][ch]);
                    if (t + 1 < L) bn = (1.f - bfu(tl.lam[j + 1][ch])) * bfu(tl.dt[j + 1][ch]);
                }
                const float w = fmaf(lam, dt, bn) * x;
                float Bv[NSL];
                ld4(&tl.B[j][NSL * half], Bv);
#pragma unroll
                for (int i = 0; i < NSL; ++i) {
                    K[i] = fmaf(ex2f(a2[i] * dt), K[i], w * Bv[i]);
                    Ks[((j + 1) * NSL + i) * NT + tid] = K[i];
                }
            }
        }
        __syncthreads();
        // ---- reverse sweep over the tile ------------------------------------------
#pragma unroll 1
        for (int j = TT - 1; j >= 0; --j) {
            const int t = t0 + j;
            float v[2 * NSL];   // dB, dC of this thread's rows
            if (t < L) {
                const float dt = bfu(tl.dt[j][ch]), x = bfu(tl.x[j][ch]), dy = bfu(tl.dy[j][ch]);
                float lam = 1.f, bn = 0.f;
                if (p.two_ep) {
                    lam = bfu(tl.lam[j][ch]);
                    if (t + 1 < L) bn = (1.f - bfu(tl.lam[j + 1][ch])) * bfu(tl.dt[j + 1][ch]);
                }
                const float sig = fmaf(lam, dt, bn), cbt = s_cb[j];
                float Bv[NSL], Cv[NSL];
                ld4(&tl.B[j][NSL * half], Bv);
                ld4(&tl.C[j][NSL * half], Cv);
                const float bxd = bn * x * dy;
                float sBG = 0.f, adr = 0.f;
#pragma unroll
                for (int i = 0; i < NSL; ++i) {
                    G[i] = fmaf(Cv[i], dy, G[i]);   // readout of K_t
                    const float kt = Ks[((j + 1) * NSL + i) * NT + tid];
                    const float kp = Ks[(j * NSL + i) * NT + tid];
                    v[NSL + i] = fmaf(dy, kt, -bxd * Bv[i]);            // dC
                    v[i] = fmaf(sig * x, G[i], -bxd * Cv[i]);          // dB
                    sBG = fmaf(Bv[i], G[i], sBG);
                    const float e = ex2f(a2[i] * dt);
                    const float dr = G[i] * e * kp;                    // drho_{t,n}
                    dA[i] = fmaf(dt, dr, dA[i]);
                    adr = fmaf(a[i], dr, adr);
                    G[i] *= e;
                }
                sBG = lane_sum<S>(sBG);
                adr = lane_sum<S>(adr);
                const float dsig = sBG * x;                 // = dgamma_t = part of dbeta_{t+1}
                const float dbn = dsig - cbt * x * dy;      // dbeta_{t+1}
                finish(dbn);                                // token t + 1 is complete
                pend_t = t;
                pend_lam = lam;
                pend_dt = dt;
                pend_dgam = dsig;
                pend_base = fmaf(lam, dsig, adr);
                if (half == 0) {
                    const float dxv = fmaf(fmaf(-bn, cbt, D), dy, sig * sBG);
                    st_io(p.dx, ix_x(p, b, t, h, 0, 0), dxv, 1);
                    dD = fmaf(dy, x, dD);
                }
            } else {
#pragma unroll
                for (int i = 0; i < 2 * NSL; ++i) v[i] = 0.f;
            }
            chan_reduce8<S>(v, lane);
            // lane l now holds value (l >> 2) & 7 (dB rows for 0..3, dC rows for 4..7) of
            // its sub-block `half` of rows, summed over the warp's channels
            red[(warp * TT + j) * 32 + ((lane >> 2) & 7) * S + half] = v[0];
        }
        __syncthreads();
        // ---- the CTA's partial dB / dC of the tile: sum over its warps in order -------
        // red[w][j][vi * S + sub]: vi < NSL -> dB row NSL sub + vi, else dC row NSL sub + vi - NSL
        for (int i = tid; i < TT * 2 * p.N; i += NT) {
            const int j = i / (2 * p.N), r = i % (2 * p.N);
            const int kind = r / p.N, n = r % p.N;           // kind 0 = dB, 1 = dC
            const int sub = n / NSL, vi = kind * NSL + n % NSL;
            const int slot = vi * S + sub;
            float s = 0.f;
            for (int w = 0; w < NW; ++w) s += red[(w * TT + j) * 32 + slot];
            const int t = t0 + j;
            if (t < L)
                bc_part[((((long long)b * p.L + t) * p.G + g) * nblk + blk) * 2 * p.N + r] = s;
        }
        __syncthreads();
    }
    // token 0: dbeta_0 = <dL/dK_{-1}, w0>; dh0 = G, dw0 = beta_0 G
    float beta0 = 0.f, db0 = 0.f;
    if (p.two_ep && L > 0)
        beta0 = (1.f - ld_io(p.lam, ix_lam(p, b, 0, h), 1)) * ld_io(p.dt, ix_dt(p, b, 0, h), 1);
#pragma unroll
    for (int i = 0; i < NSL; ++i) {
        const long long ii = ix_st(p, b, h, NSL * half + i, 0);
        if (p.dh0) p.dh0[ii] = G[i];
        if (p.dw0) p.dw0[ii] = beta0 * G[i];
        if (p.w0) db0 = fmaf(G[i], p.w0[ii], db0);
    }
    db0 = lane_sum<S>(db0);
    finish(db0);
    // per-(b, h) partial parameter gradients: sum_t dt drho per row, <dy, x>
#pragma unroll
    for (int i = 0; i < NSL; ++i)
        par_part[((long long)b * p.H + h) * (p.N + 1) + NSL * half + i] = dA[i];
    if (half == 0) par_part[((long long)b * p.H + h) * (p.N + 1) + p.N] = dD;
}

// dB / dC of a group: the fixed-order sum of its CTAs' partials.
__global__ void k_m1_bc_sum(Params p, const float *bc_part) {
    const int nblk = p.hpg / m1::CPB;
    const long long total = (long long)p.Bsz * p.L * p.G * 2 * p.N;
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
         i += (long long)gridDim.x * blockDim.x) {
        const int r = (int)(i % (2 * p.N));
        const long long bt = i / (2 * p.N);
        const int g = (int)(bt % p.G);
        const long long btt = bt / p.G;
        const int t = (int)(btt % p.L), b = (int)(btt / p.L);
        float s = 0.f;
        for (int k = 0; k < nblk; ++k) s += bc_part[(bt * nblk + k) * 2 * p.N + r];
        const int n = r % p.N;
        if (r < p.N)
            st_io(p.dBm, ix_B(p, b, t, g, 0, n), s, 1);
        else
            st_io(p.dCm, ix_C(p, b, t, g, 0, n), s, 1);
    }
}

// dA_log = a sum_{b, t} dt drho, dD = sum <dy, x> (fixed order over batch rows).
__global__ void k_m1_params(Params p, const float *par_part) {
    for (int h = blockIdx.x * blockDim.x + threadIdx.x; h < p.H; h += gridDim.x * blockDim.x) {
        float sd = 0.f;
        for (int b = 0; b < p.Bsz; ++b) sd += par_part[((long long)b * p.H + h) * (p.N + 1) + p.N];
        if (p.dD) p.dD[h] = sd;
        for (int k = 0; k < p.ndec; ++k) {
            float s = 0.f;
            for (int b = 0; b < p.Bsz; ++b)
                for (int n = 0; n < p.N; ++n)
                    if (!p.per_coord || n == k) s += par_part[((long long)b * p.H + h) * (p.N + 1) + n];
            p.dA_log[h * p.ndec + k] = -expf(__ldg(p.A_log + h * p.ndec + k)) * s;
        }
    }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
// Shapes the channel scan takes (pointer alignment and strides included).
bool m1_supported(const Params &p) {
    auto al16 = [](const void *ptr) { return ptr == nullptr || ((uintptr_t)ptr & 15) == 0; };
    auto m8 = [](long long s) { return s % 8 == 0; };
    return p.bf16 && p.P == 1 && p.R == 1 && p.O == 1 && p.np == 0 && (p.N == 8 || p.N == 16) &&
           p.hpg % m1::CPB == 0 && p.L > 0 && al16(p.x) && al16(p.dt) && al16(p.lam) &&
           al16(p.y) && al16(p.dy) && al16(p.Bm) && al16(p.Cm) && p.sx[2] == 1 && p.sy[2] == 1 &&
           p.sdt[2] == 1 && (!p.two_ep || p.slam[2] == 1) && m8(p.sx[1]) && m8(p.sx[0]) &&
           m8(p.sy[1]) && m8(p.sy[0]) && m8(p.sdt[1]) && m8(p.sdt[0]) &&
           (!p.two_ep || (m8(p.slam[1]) && m8(p.slam[0]))) && m8(p.sB[0]) && m8(p.sB[1]) &&
           m8(p.sB[2]) && m8(p.sC[0]) && m8(p.sC[1]) && m8(p.sC[2]);
}

// Workspace of the channel scan (floats): the kept states [B][H][tiles][N], the
// dB / dC partials [B][L][G][H / G / 64][2 N] and the parameter partials
// [B][H][N + 1].
size_t m1_kept_floats(long long B, long long L, long long H, int N) {
    return (size_t)B * H * ((L + m1::TT - 1) / m1::TT) * N;
}
size_t m1_part_floats(long long B, long long L, long long H, int N) {
    return (size_t)B * L * (H / m1::CPB) * 2 * N + (size_t)B * H * (N + 1);
}

cudaError_t m1_forward(const Params &p, float *kept, cudaStream_t st) {
    const dim3 grid(p.H / m1::CPB, p.Bsz);
    if (p.N == 16) {
        k_m1_fwd<4><<<grid, 256, 0, st>>>(p, kept);
    } else {
        k_m1_fwd<2><<<grid, 128, 0, st>>>(p, kept);
    }
    profile_mark(st, "k_m1_fwd");
    return cudaGetLastError();
}

template <int S>
static size_t m1_bwd_smem() {
    constexpr int NT = 64 * S;
    return 2 * sizeof(m1::Tile) + (size_t)((m1::TT + 1) * m1::NSL * NT + (NT / 32) * m1::TT * 32 +
                                           m1::TT) * sizeof(float);
}

// Backward: `kept` holds the states a training forward kept (or is filled
// here by a forward that writes them and nothing else).
cudaError_t m1_backward(const Params &p, float *kept, bool kept_ready, float *part,
                        cudaStream_t st) {
    cudaError_t e;
    if (!kept_ready) {
        Params pf = p;
        pf.y = nullptr;
        pf.hT = nullptr;
        pf.wT = nullptr;
        if ((e = m1_forward(pf, kept, st)) != cudaSuccess) return e;
    }
    float *bc_part = part;
    float *par_part = part + (size_t)p.Bsz * p.L * (p.H / m1::CPB) * 2 * p.N;
    const dim3 grid(p.H / m1::CPB, p.Bsz);
    if (p.N == 16) {
        const size_t sm = m1_bwd_smem<4>();
        if ((e = cudaFuncSetAttribute(k_m1_bwd<4>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      (int)sm)) != cudaSuccess)
            return e;
        k_m1_bwd<4><<<grid, 256, sm, st>>>(p, kept, bc_part, par_part);
    } else {
        const size_t sm = m1_bwd_smem<2>();
        if ((e = cudaFuncSetAttribute(k_m1_bwd<2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      (int)sm)) != cudaSuccess)
            return e;
        k_m1_bwd<2><<<grid, 128, sm, st>>>(p, kept, bc_part, par_part);
    }
    profile_mark(st, "k_m1_bwd");
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const long long tot = (long long)p.Bsz * p.L * p.G * 2 * p.N;
    int blocks = (int)((tot + 255) / 256);
    if (blocks > 148 * 16) blocks = 148 * 16;
    k_m1_bc_sum<<<blocks, 256, 0, st>>>(p, bc_part);
    profile_mark(st, "k_m1_bc_sum");
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    k_m1_params<<<(p.H + 127) / 128, 128, 0, st>>>(p, par_part);
    profile_mark(st, "k_m1_params");
    return cudaGetLastError();
}

}  // namespace ssm
