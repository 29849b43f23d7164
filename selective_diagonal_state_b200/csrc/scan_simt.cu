// Recurrent (SIMT) selective diagonal scan: forward and backward for every mode
// (real per-coordinate or per-head decay, 2x2 rotation pairs, two-endpoint
// writes, rank-R routing).  fp32 state in registers, one CTA per (batch row,
// HC heads); inputs of T tokens at a time are staged in shared memory.
//
// Arithmetic (the recurrence of "When a Diagonal State Is Not Enough",
// sungsoo.github.io Part 01 / Part 03, with the two-endpoint write of Part 05)
// is run in the equivalent "pre-state" form
//      K_t = A_t K_{t-1} + sigma_t W_t,   sigma_t = gamma_t + beta_{t+1},
//      K_t = H_t + beta_{t+1} W_t,   K_{-1} = h0 + beta_0 w0,
//      y_t = C_t K_t - beta_{t+1} (C_t B_t) u_t + D u_t,
// which costs one multiply-add per state element and step (beta_L = 0, so
// K_{L-1} = H_{L-1}).
//
// Backward (reverse mode of the same form):
//   sweep 1 (forward in t) recomputes K_t and stores dC_t = dy_t H_t^T per head;
//   sweep 2 (reverse in t) runs Gbar_t = C_t^T dy_t + A_{t+1}^T Gbar_{t+1},
//     storing sum_p Gbar u^T and writing dx;
//   the decay gradients use, for every state mode m, the identity
//     dL/d(log-transition of step tau) = sum_{t >= tau} (X_t - Y_t),
//     X_t = conj(c_t) . sum_p dy_t,p K_t,p,   Y_t = sigma_t b_t . conj(sum_p u_t,p Gbar_t,p)
//   (complex for rotation pairs: real part -> decay, minus imaginary part ->
//   angle), so no per-step state has to be kept.
#include "common.cuh"

namespace ssm {

constexpr int MAXT = 256;

__device__ __forceinline__ float neg_exp(float v) { return -expf(v); }

// ------------------------------------------------------------------------
// shared-memory plan (floats) common to the scan kernels
// ------------------------------------------------------------------------
struct Smem {
    float *a, *w;             // [HC][ndec] decay rates a = -exp(A_log); [HC][np] theta
    float *dt, *lam;          // [HC][T+1]
    float *sig, *bn;          // [HC][T]  sigma_t, beta_{t+1}
    float *coef;              // [HC][T][NSL]  decay per real slot, (e cos, e sin) per pair
    float *Bp, *Cp;           // [NGL][T][R][NSL], [NGL][T][O][NSL]
    float *u, *dy;            // [HC][T][R][PP], [HC][T][O][PP]
    float *corr;              // [HC][T][O][R]   -beta_{t+1} (C_t B_t)[o][r]   (or M for bwd)
    float *red;               // reduction buffer (kernel specific)
    float *misc;              // [HC][T][4]
    float *zc;                // [HC][T][NSL]  ZOH write coefficient per slot (re, im per pair)
    int *slot;                // [N] slot of each state row
};

// Threads cover a (rows x width) loop as (tid / W, tid % W) with W the
// smallest power of two >= min(width, blockDim): no division per element.
struct Lanes2D {
    int tx, ty, W, ny;
};
__device__ __forceinline__ Lanes2D lanes2d(int width) {
    const int nthr = blockDim.x;
    int W = 1;
    while (W < width && W < nthr) W <<= 1;
    Lanes2D l;
    l.W = W;
    l.tx = threadIdx.x & (W - 1);
    l.ty = threadIdx.x / W;
    l.ny = nthr / W;
    return l;
}

template <int NR, int NPR>
__device__ __forceinline__ int ngl_of(const Params &p, int hbase, int HC) {
    int hl = min(hbase + HC, p.H) - 1;
    return hl / p.hpg - hbase / p.hpg + 1;
}

// Lay the arrays out from `base` (16-byte aligned each); returns the float
// count up to the start of the reduction buffer.  The host calls it with a
// null base to size the allocation.
__host__ __device__ inline size_t carve(Smem &s, float *base, const Params &p, int NSL, int NGL,
                                        bool with_dy) {
    const Geometry &g = p.geo;
    size_t off = 0;
    auto take = [&](size_t n) {
        float *r = base ? base + off : nullptr;
        off += (n + 3) & ~size_t(3);
        return r;
    };
    s.a = take((size_t)g.HC * p.ndec);
    s.w = take((size_t)g.HC * (p.np > 0 ? p.np : 1));
    s.dt = take((size_t)g.HC * (g.T + 1));
    s.lam = take((size_t)g.HC * (g.T + 1));
    s.sig = take((size_t)g.HC * g.T);
    s.bn = take((size_t)g.HC * g.T);
    s.coef = take((size_t)g.HC * g.T * NSL);
    s.Bp = take((size_t)NGL * g.T * p.R * NSL);
    s.Cp = take((size_t)NGL * g.T * p.O * NSL);
    s.u = take((size_t)g.HC * g.T * p.R * g.PP);
    s.dy = with_dy ? take((size_t)g.HC * g.T * p.O * g.PP) : nullptr;
    s.corr = take((size_t)g.HC * g.T * p.O * p.R);
    s.misc = take((size_t)g.HC * g.T * 4);
    s.zc = take(p.zoh ? (size_t)g.HC * g.T * NSL : 0);
    s.slot = reinterpret_cast<int *>(take((size_t)p.N));
    s.red = base ? base + off : nullptr;
    return off;
}

__host__ inline size_t smem_floats(const Params &p, int NSL, int NGL, size_t red_floats,
                                   bool with_dy) {
    Smem s;
    return carve(s, nullptr, p, NSL, NGL, with_dy) + red_floats;
}

// Load tokens [t0, t0+T) of this CTA's heads into shared memory and derive
// the per-step coefficients.  `reverse_coef` is unused (coefficients are those
// of each step t itself).  Padding slots stay zero.
template <int NR, int NPR>
__device__ void stage_block(const Params &p, Smem &s, int b, int hbase, int gbase, int NGL,
                            int t0, bool with_dy) {
    const Geometry &g = p.geo;
    const int T = g.T, HC = g.HC, NQ = g.NQ, PP = g.PP;
    constexpr int NS = NR + 2 * NPR;
    const int NSL = NQ * NS;
    const int tid = threadIdx.x, nthr = blockDim.x;
    // dt, lambda for t0 .. t0+T (one past the block for beta_{t+1})
    for (int i = tid; i < HC * (T + 1); i += nthr) {
        int hc = i / (T + 1), tt = i - hc * (T + 1), h = hbase + hc, t = t0 + tt;
        float dv = 0.f, lv = 1.f;
        if (h < p.H && t < p.L) {
            dv = ld_io(p.dt, ix_dt(p, b, t, h), p.bf16);
            if (p.two_ep) lv = ld_io(p.lam, ix_lam(p, b, t, h), p.bf16);
        }
        s.dt[i] = dv;
        s.lam[i] = lv;
    }
    {
        const Lanes2D l = lanes2d(p.N);
        for (int gl = 0; gl < NGL; ++gl) {
            const int gg = gbase + gl;
            for (int tt = l.ty; tt < T; tt += l.ny) {
                const int t = t0 + tt;
                const bool ok = gg < p.G && t < p.L;
                for (int r = 0; r < p.R; ++r) {
                    float *dst = s.Bp + ((gl * T + tt) * p.R + r) * NSL;
                    for (int n = l.tx; n < p.N; n += l.W)
                        dst[s.slot[n]] = ok ? ld_io(p.Bm, ix_B(p, b, t, gg, r, n), p.bf16) : 0.f;
                }
                for (int o = 0; o < p.O; ++o) {
                    float *dst = s.Cp + ((gl * T + tt) * p.O + o) * NSL;
                    for (int n = l.tx; n < p.N; n += l.W)
                        dst[s.slot[n]] = ok ? ld_io(p.Cm, ix_C(p, b, t, gg, o, n), p.bf16) : 0.f;
                }
            }
        }
    }
    {
        const Lanes2D l = lanes2d(PP);
        for (int hc = 0; hc < HC; ++hc) {
            const int h = hbase + hc;
            for (int tt = l.ty; tt < T; tt += l.ny) {
                const int t = t0 + tt;
                const bool ok = h < p.H && t < p.L;
                for (int r = 0; r < p.R; ++r) {
                    float *dst = s.u + ((hc * T + tt) * p.R + r) * PP;
                    for (int q = l.tx; q < PP; q += l.W)
                        dst[q] = (ok && q < p.P) ? ld_io(p.x, ix_x(p, b, t, h, r, q), p.bf16) : 0.f;
                }
                if (with_dy) {
                    for (int o = 0; o < p.O; ++o) {
                        float *dst = s.dy + ((hc * T + tt) * p.O + o) * PP;
                        for (int q = l.tx; q < PP; q += l.W)
                            dst[q] = (ok && q < p.P) ? ld_io(p.dy, ix_y(p, b, t, h, o, q), p.bf16)
                                                     : 0.f;
                    }
                }
            }
        }
    }
    __syncthreads();
    for (int i = tid; i < HC * T; i += nthr) {
        int hc = i / T, tt = i - hc * T, t = t0 + tt;
        float dv = s.dt[hc * (T + 1) + tt], lv = s.lam[hc * (T + 1) + tt];
        float bnext = 0.f;
        if (t + 1 < p.L) bnext = (1.f - s.lam[hc * (T + 1) + tt + 1]) * s.dt[hc * (T + 1) + tt + 1];
        s.sig[i] = p.zoh ? 1.f : lv * dv + bnext;   // the ZOH write is scaled per mode
        s.bn[i] = bnext;
    }
    const int nmode = p.nr + p.np;
    {
        const Lanes2D l = lanes2d(nmode);
        for (int hc = 0; hc < HC; ++hc) {
            const int h = hbase + hc;
            for (int tt = l.ty; tt < T; tt += l.ny) {
                const float dv = s.dt[hc * (T + 1) + tt];
                const bool tok_ok = h < p.H && t0 + tt < p.L;
                float *cf = s.coef + (hc * T + tt) * NSL;
                for (int m = l.tx; m < nmode; m += l.W) {
                    const float a = s.a[hc * p.ndec + (p.per_coord ? m : 0)];
                    if (p.zoh) {
                        // Z = dt phi1(dt a + i phi): the exact write of a held input
                        float phi = 0.f;
                        if (m >= p.nr) {
                            const int j = m - p.nr;
                            phi = p.angle_tok ? (tok_ok ? p.theta[ix_th(p, b, t0 + tt, h, j)] : 0.f)
                                              : dv * s.w[hc * (p.np > 0 ? p.np : 1) + j];
                        }
                        float f1r, f1i, fdr, fdi;
                        zoh_phi(dv * a, phi, f1r, f1i, fdr, fdi);
                        float *zz = s.zc + (hc * T + tt) * NSL;
                        if (m < p.nr) {
                            zz[s.slot[m]] = dv * f1r;
                        } else {
                            const int sl = s.slot[p.nr + 2 * (m - p.nr)];
                            zz[sl] = dv * f1r;
                            zz[sl + 1] = dv * f1i;
                        }
                    }
                    if (m < p.nr) {
                        cf[s.slot[m]] = expf(m < p.nst ? a : dv * a);   // static rows: e^{a}
                    } else {
                        const int j = m - p.nr;
                        float e = expf(dv * a), sn, cs;
                        // angle of step t: per token, or the pair's frequency times dt_t
                        const float phi =
                            p.angle_tok ? (tok_ok ? p.theta[ix_th(p, b, t0 + tt, h, j)] : 0.f)
                                        : dv * s.w[hc * (p.np > 0 ? p.np : 1) + j];
                        sincosf(phi, &sn, &cs);
                        const int sl = s.slot[p.nr + 2 * j];
                        cf[sl] = e * cs;
                        cf[sl + 1] = e * sn;
                    }
                }
            }
        }
    }
    // M_t[o][r] = sum_n C[o][n] B[n][r] (callers scale by beta_{t+1})
    for (int i = tid; i < HC * T * p.O * p.R; i += nthr) {
        int r = i % p.R, o = (i / p.R) % p.O, tt = (i / (p.R * p.O)) % T, hc = i / (p.R * p.O * T);
        int h = hbase + hc, gl = (h < p.H ? h : hbase) / p.hpg - gbase;
        const float *cp = s.Cp + ((gl * T + tt) * p.O + o) * NSL;
        const float *bp = s.Bp + ((gl * T + tt) * p.R + r) * NSL;
        float acc = 0.f;
        for (int k = 0; k < NSL; ++k) acc = fmaf(cp[k], bp[k], acc);
        s.corr[i] = acc;  // plain M; callers scale by beta_{t+1}
    }
    __syncthreads();
}

template <int NR, int NPR>
__device__ void init_rates(const Params &p, Smem &s, int hbase, int NSL, int NGL) {
    const Geometry &g = p.geo;
    for (int i = threadIdx.x; i < g.HC * p.ndec; i += blockDim.x) {
        int hc = i / p.ndec, k = i % p.ndec, h = min(hbase + hc, p.H - 1);
        s.a[i] = neg_exp(p.A_log[h * p.ndec + k]);
    }
    for (int i = threadIdx.x; i < g.HC * p.np; i += blockDim.x) {
        int hc = i / p.np, j = i % p.np, h = min(hbase + hc, p.H - 1);
        s.w[i] = p.angle_tok ? 0.f : p.theta[h * p.np + j];
    }
    for (int n = threadIdx.x; n < p.N; n += blockDim.x) s.slot[n] = slot_of<NR, NPR>(n, p.nr, g.NQ);
    // padding slots must read as zero for the whole kernel
    for (int i = threadIdx.x; i < g.HC * g.T * NSL; i += blockDim.x) s.coef[i] = 0.f;
    if (p.zoh)
        for (int i = threadIdx.x; i < g.HC * g.T * NSL; i += blockDim.x) s.zc[i] = 0.f;
    for (int i = threadIdx.x; i < NGL * g.T * p.R * NSL; i += blockDim.x) s.Bp[i] = 0.f;
    for (int i = threadIdx.x; i < NGL * g.T * p.O * NSL; i += blockDim.x) s.Cp[i] = 0.f;
    __syncthreads();
}

// one step of K_t = A_t K_{t-1} + w over this thread's slots
template <int NR, int NPR>
__device__ __forceinline__ void step_fwd(float (&K)[NR + 2 * NPR], const float *cf,
                                         const float (&w)[NR + 2 * NPR]) {
#pragma unroll
    for (int i = 0; i < NR; ++i) K[i] = fmaf(cf[i], K[i], w[i]);
#pragma unroll
    for (int j = 0; j < NPR; ++j) {
        const float ec = cf[NR + 2 * j], es = cf[NR + 2 * j + 1];
        const float kr = K[NR + 2 * j], ki = K[NR + 2 * j + 1];
        K[NR + 2 * j] = fmaf(ec, kr, fmaf(-es, ki, w[NR + 2 * j]));
        K[NR + 2 * j + 1] = fmaf(es, kr, fmaf(ec, ki, w[NR + 2 * j + 1]));
    }
}
// w <- Z (.) w (ZOH write; complex product on a pair) and its transpose
template <int NR, int NPR>
__device__ __forceinline__ void zoh_apply(float (&w)[NR + 2 * NPR], const float *zz) {
#pragma unroll
    for (int i = 0; i < NR; ++i) w[i] *= zz[i];
#pragma unroll
    for (int j = 0; j < NPR; ++j) {
        const float zr = zz[NR + 2 * j], zi = zz[NR + 2 * j + 1];
        const float wr = w[NR + 2 * j], wi = w[NR + 2 * j + 1];
        w[NR + 2 * j] = fmaf(zr, wr, -zi * wi);
        w[NR + 2 * j + 1] = fmaf(zi, wr, zr * wi);
    }
}
template <int NR, int NPR>
__device__ __forceinline__ void zoh_apply_T(float (&g)[NR + 2 * NPR], const float *zz) {
#pragma unroll
    for (int i = 0; i < NR; ++i) g[i] *= zz[i];
#pragma unroll
    for (int j = 0; j < NPR; ++j) {
        const float zr = zz[NR + 2 * j], zi = zz[NR + 2 * j + 1];
        const float gr = g[NR + 2 * j], gi = g[NR + 2 * j + 1];
        g[NR + 2 * j] = fmaf(zr, gr, zi * gi);
        g[NR + 2 * j + 1] = fmaf(-zi, gr, zr * gi);
    }
}
// G <- A_t^T G
template <int NR, int NPR>
__device__ __forceinline__ void step_adj(float (&Gv)[NR + 2 * NPR], const float *cf) {
#pragma unroll
    for (int i = 0; i < NR; ++i) Gv[i] *= cf[i];
#pragma unroll
    for (int j = 0; j < NPR; ++j) {
        const float ec = cf[NR + 2 * j], es = cf[NR + 2 * j + 1];
        const float gr = Gv[NR + 2 * j], gi = Gv[NR + 2 * j + 1];
        Gv[NR + 2 * j] = fmaf(ec, gr, es * gi);
        Gv[NR + 2 * j + 1] = fmaf(-es, gr, ec * gi);
    }
}

template <int NS>
__device__ __forceinline__ void ld_slots(float (&dst)[NS], const float *src) {
#pragma unroll
    for (int i = 0; i < NS; i += 4) {
        float4 v = *reinterpret_cast<const float4 *>(src + i);
        dst[i] = v.x;
        dst[i + 1] = v.y;
        dst[i + 2] = v.z;
        dst[i + 3] = v.w;
    }
}

struct Lane {
    int pl, q, hc, h, b, hbase, gbase, gl, NGL;
    bool hv;
};

template <int NR, int NPR>
__device__ __forceinline__ Lane lane_of(const Params &p) {
    const Geometry &g = p.geo;
    Lane l;
    int tid = threadIdx.x;
    l.pl = tid % g.PP;
    l.q = (tid / g.PP) % g.NQ;
    l.hc = tid / (g.PP * g.NQ);
    l.b = blockIdx.y;
    l.hbase = blockIdx.x * g.HC;
    l.h = l.hbase + l.hc;
    l.hv = l.h < p.H;
    l.gbase = l.hbase / p.hpg;
    l.NGL = ngl_of<NR, NPR>(p, l.hbase, g.HC);
    l.gl = (l.hv ? l.h : l.hbase) / p.hpg - l.gbase;
    return l;
}

// ------------------------------------------------------------------------
// forward
// ------------------------------------------------------------------------
template <int NR, int NPR, int RM>
__global__ void __launch_bounds__(MAXT) k_fwd(Params p) {
    if (gated_off(p)) return;
    extern __shared__ __align__(16) float smem[];
    constexpr int NS = NR + 2 * NPR;
    const Geometry &g = p.geo;
    const int T = g.T, NQ = g.NQ, PP = g.PP, HC = g.HC, NSL = NQ * NS;
    const Lane ln = lane_of<NR, NPR>(p);
    Smem s;
    carve(s, smem, p, NSL, ln.NGL, false);
    init_rates<NR, NPR>(p, s, ln.hbase, NSL, ln.NGL);
    const bool act = ln.hv && ln.pl < p.P;

    // K_{-1} = h0 + beta_0 w0
    float K[NS];
    {
        float beta0 = 0.f;
        if (ln.hv && p.two_ep && p.L > 0)
            beta0 = (1.f - ld_io(p.lam, ix_lam(p, ln.b, 0, ln.h), p.bf16)) *
                    ld_io(p.dt, ix_dt(p, ln.b, 0, ln.h), p.bf16);
#pragma unroll
        for (int sl = 0; sl < NS; ++sl) {
            int n = row_of<NR, NPR>(ln.q, sl, p.nr, p.np, NQ);
            float v = 0.f;
            if (act && n >= 0) {
                if (p.h0) v = p.h0[ix_st(p, ln.b, ln.h, n, ln.pl)];
                if (p.w0) v = fmaf(beta0, p.w0[ix_st(p, ln.b, ln.h, n, ln.pl)], v);
            }
            K[sl] = v;
        }
    }
    float Wlast[NS];
#pragma unroll
    for (int sl = 0; sl < NS; ++sl) Wlast[sl] = 0.f;

    for (int t0 = 0; t0 < p.L; t0 += T) {
        stage_block<NR, NPR>(p, s, ln.b, ln.hbase, ln.gbase, ln.NGL, t0, false);
        const int tn = min(T, p.L - t0);
        for (int tt = 0; tt < tn; ++tt) {
            const float sig = s.sig[ln.hc * T + tt];
            float su[RM];
#pragma unroll
            for (int r = 0; r < RM; ++r)
                su[r] = r < p.R ? s.u[((ln.hc * T + tt) * p.R + r) * PP + ln.pl] : 0.f;
            float w[NS];
#pragma unroll
            for (int sl = 0; sl < NS; ++sl) w[sl] = 0.f;
#pragma unroll
            for (int r = 0; r < RM; ++r) {
                if (r < p.R) {
                    float bb[NS];
                    ld_slots<NS>(bb, s.Bp + ((ln.gl * T + tt) * p.R + r) * NSL + ln.q * NS);
#pragma unroll
                    for (int sl = 0; sl < NS; ++sl) w[sl] = fmaf(bb[sl], su[r], w[sl]);
                }
            }
            if (t0 + tt == p.L - 1) {
#pragma unroll
                for (int sl = 0; sl < NS; ++sl) Wlast[sl] = w[sl];
            }
            if (p.zoh) {
                float zz[NS];
                ld_slots<NS>(zz, s.zc + (ln.hc * T + tt) * NSL + ln.q * NS);
                zoh_apply<NR, NPR>(w, zz);
            } else {
#pragma unroll
                for (int sl = 0; sl < NS; ++sl) w[sl] *= sig;
            }
            float cf[NS];
            ld_slots<NS>(cf, s.coef + (ln.hc * T + tt) * NSL + ln.q * NS);
            step_fwd<NR, NPR>(K, cf, w);
#pragma unroll
            for (int o = 0; o < RM; ++o) {
                if (o < p.O) {
                    float cc[NS];
                    ld_slots<NS>(cc, s.Cp + ((ln.gl * T + tt) * p.O + o) * NSL + ln.q * NS);
                    float acc = 0.f;
#pragma unroll
                    for (int sl = 0; sl < NS; ++sl) acc = fmaf(cc[sl], K[sl], acc);
                    s.red[(((ln.hc * T + tt) * p.O + o) * NQ + ln.q) * PP + ln.pl] = acc;
                }
            }
        }
        __syncthreads();
        // y = C K - beta_{t+1} M u + D u, summed over the row groups (not written by a
        // state-only forward)
        const Lanes2D l2 = lanes2d(p.P);
        for (int row = l2.ty; p.y && row < HC * T * p.O; row += l2.ny)
        for (int q = l2.tx; q < p.P; q += l2.W) {
            const int o = row % p.O, tt = (row / p.O) % T, hc = row / (p.O * T);
            int h = ln.hbase + hc, t = t0 + tt;
            if (h >= p.H || t >= p.L) continue;
            float v = 0.f;
            for (int k = 0; k < NQ; ++k) v += s.red[(((hc * T + tt) * p.O + o) * NQ + k) * PP + q];
            const float bnx = s.bn[hc * T + tt];
            for (int r = 0; r < p.R; ++r)
                v = fmaf(-bnx * s.corr[((hc * T + tt) * p.O + o) * p.R + r],
                         s.u[((hc * T + tt) * p.R + r) * PP + q], v);
            if (p.O == p.R) v = fmaf(p.D[h], s.u[((hc * T + tt) * p.R + o) * PP + q], v);
            st_io(p.y, ix_y(p, ln.b, t, h, o, q), v, p.bf16);
        }
        __syncthreads();
    }
    if (act) {
#pragma unroll
        for (int sl = 0; sl < NS; ++sl) {
            int n = row_of<NR, NPR>(ln.q, sl, p.nr, p.np, NQ);
            if (n < 0) continue;
            if (p.hT) p.hT[ix_st(p, ln.b, ln.h, n, ln.pl)] = K[sl];
            if (p.wT) {
                float v = p.L > 0 ? Wlast[sl] : (p.w0 ? p.w0[ix_st(p, ln.b, ln.h, n, ln.pl)] : 0.f);
                p.wT[ix_st(p, ln.b, ln.h, n, ln.pl)] = v;
            }
        }
    }
}

// Write `v` (this lane's share of a K-value xreduce) into red[...][k].
template <int K, int S>
__device__ __forceinline__ void put_reduced(float *dst, const float (&v)[K], int lane_in_s) {
    if constexpr (K >= S) {
        constexpr int KS = K / S;
#pragma unroll
        for (int i = 0; i < KS; ++i) dst[lane_in_s * KS + i] = v[i];
    } else {
        constexpr int SK = S / K;
        if (lane_in_s % SK == 0) dst[lane_in_s / SK] = v[0];
    }
}

// ------------------------------------------------------------------------
// backward sweep 1: recompute K_t forward, store dC_t = dy_t H_t^T per head
// red layout: [HC][T][NWP][NQ][RM*NS]
// ------------------------------------------------------------------------
template <int NR, int NPR, int RM, int S>
__global__ void __launch_bounds__(MAXT) k_bwd_sweep1(Params p) {
    if (gated_off(p)) return;
    extern __shared__ __align__(16) float smem[];
    constexpr int NS = NR + 2 * NPR;
    constexpr int KV = RM * NS;
    const Geometry &g = p.geo;
    const int T = g.T, NQ = g.NQ, PP = g.PP, HC = g.HC, NSL = NQ * NS;
    const int NWP = PP > 32 ? PP / 32 : 1;
    const Lane ln = lane_of<NR, NPR>(p);
    Smem s;
    carve(s, smem, p, NSL, ln.NGL, true);
    init_rates<NR, NPR>(p, s, ln.hbase, NSL, ln.NGL);
    const bool act = ln.hv && ln.pl < p.P;
    const int lane_in_s = S > 1 ? (ln.pl % S) : 0;
    const int wp = S > 1 ? ln.pl / S : 0;

    float K[NS];
    {
        float beta0 = 0.f;
        if (ln.hv && p.two_ep && p.L > 0)
            beta0 = (1.f - ld_io(p.lam, ix_lam(p, ln.b, 0, ln.h), p.bf16)) *
                    ld_io(p.dt, ix_dt(p, ln.b, 0, ln.h), p.bf16);
#pragma unroll
        for (int sl = 0; sl < NS; ++sl) {
            int n = row_of<NR, NPR>(ln.q, sl, p.nr, p.np, NQ);
            float v = 0.f;
            if (act && n >= 0) {
                if (p.h0) v = p.h0[ix_st(p, ln.b, ln.h, n, ln.pl)];
                if (p.w0) v = fmaf(beta0, p.w0[ix_st(p, ln.b, ln.h, n, ln.pl)], v);
            }
            K[sl] = v;
        }
    }
    for (int t0 = 0; t0 < p.L; t0 += T) {
        stage_block<NR, NPR>(p, s, ln.b, ln.hbase, ln.gbase, ln.NGL, t0, true);
        const int tn = min(T, p.L - t0);
        for (int tt = 0; tt < tn; ++tt) {
            const float sig = s.sig[ln.hc * T + tt], bnx = s.bn[ln.hc * T + tt];
            float w[NS];
#pragma unroll
            for (int sl = 0; sl < NS; ++sl) w[sl] = 0.f;
#pragma unroll
            for (int r = 0; r < RM; ++r) {
                if (r < p.R) {
                    const float ur = s.u[((ln.hc * T + tt) * p.R + r) * PP + ln.pl];
                    float bb[NS];
                    ld_slots<NS>(bb, s.Bp + ((ln.gl * T + tt) * p.R + r) * NSL + ln.q * NS);
#pragma unroll
                    for (int sl = 0; sl < NS; ++sl) w[sl] = fmaf(bb[sl], ur, w[sl]);
                }
            }
            float cf[NS];
            ld_slots<NS>(cf, s.coef + (ln.hc * T + tt) * NSL + ln.q * NS);
            float ws[NS];
#pragma unroll
            for (int sl = 0; sl < NS; ++sl) ws[sl] = w[sl] * sig;
            if (p.zoh) {
                float zz[NS];
                ld_slots<NS>(zz, s.zc + (ln.hc * T + tt) * NSL + ln.q * NS);
                zoh_apply<NR, NPR>(ws, zz);
            }
            step_fwd<NR, NPR>(K, cf, ws);
            // H_t = K_t - beta_{t+1} W_t ; values dy[o,p] * H[n,p]
            float v[KV];
#pragma unroll
            for (int o = 0; o < RM; ++o) {
                const float dyo = o < p.O ? s.dy[((ln.hc * T + tt) * p.O + o) * PP + ln.pl] : 0.f;
#pragma unroll
                for (int sl = 0; sl < NS; ++sl) v[o * NS + sl] = dyo * fmaf(-bnx, w[sl], K[sl]);
            }
            xreduce<KV, S>(v, lane_in_s);
            put_reduced<KV, S>(s.red + (((ln.hc * T + tt) * NWP + wp) * NQ + ln.q) * KV, v,
                               lane_in_s);
        }
        __syncthreads();
        const Lanes2D l2 = lanes2d(p.N);
        for (int row = l2.ty; row < HC * T * p.O; row += l2.ny)
        for (int n = l2.tx; n < p.N; n += l2.W) {
            const int o = row % p.O, tt = (row / p.O) % T, hc = row / (p.O * T);
            int h = ln.hbase + hc, t = t0 + tt;
            if (h >= p.H || t >= p.L) continue;
            int sl = s.slot[n];
            int q = sl / NS, k = o * NS + sl % NS;
            float acc = 0.f;
            for (int w2 = 0; w2 < NWP; ++w2) acc += s.red[(((hc * T + tt) * NWP + w2) * NQ + q) * KV + k];
            p.ws_dC[ix_wsk(p, ln.b, t, h, o, p.O, n)] = acc;
        }
        __syncthreads();
    }
}

// ------------------------------------------------------------------------
// backward sweep 2: reverse adjoint scan.
// red layout: part A [HC][T][NWP][NQ][RM*NS] (sum_p G u), then
//             part B [HC][T][RM][NQ][PP]      (sum over own rows of B G)
// ------------------------------------------------------------------------
template <int NR, int NPR, int RM, int S>
__global__ void __launch_bounds__(MAXT) k_bwd_sweep2(Params p) {
    if (gated_off(p)) return;
    extern __shared__ __align__(16) float smem[];
    constexpr int NS = NR + 2 * NPR;
    constexpr int KV = RM * NS;
    const Geometry &g = p.geo;
    const int T = g.T, NQ = g.NQ, PP = g.PP, HC = g.HC, NSL = NQ * NS;
    const int NWP = PP > 32 ? PP / 32 : 1;
    const Lane ln = lane_of<NR, NPR>(p);
    Smem s;
    carve(s, smem, p, NSL, ln.NGL, true);
    init_rates<NR, NPR>(p, s, ln.hbase, NSL, ln.NGL);
    float *redA = s.red;
    float *redB = s.red + (size_t)HC * T * NWP * NQ * KV;
    const bool act = ln.hv && ln.pl < p.P;
    const int lane_in_s = S > 1 ? (ln.pl % S) : 0;
    const int wp = S > 1 ? ln.pl / S : 0;

    float Gv[NS];
#pragma unroll
    for (int sl = 0; sl < NS; ++sl) Gv[sl] = 0.f;
    float cf0[NS];  // coefficients of step 0 (applied after the last iteration)
#pragma unroll
    for (int sl = 0; sl < NS; ++sl) cf0[sl] = 0.f;

    const int nblk = (p.L + T - 1) / T;
    for (int bi = nblk - 1; bi >= 0; --bi) {
        const int t0 = bi * T;
        stage_block<NR, NPR>(p, s, ln.b, ln.hbase, ln.gbase, ln.NGL, t0, true);
        const int tn = min(T, p.L - t0);
        for (int tt = tn - 1; tt >= 0; --tt) {
            // G += C_t^T dy_t
#pragma unroll
            for (int o = 0; o < RM; ++o) {
                if (o < p.O) {
                    const float dyo = s.dy[((ln.hc * T + tt) * p.O + o) * PP + ln.pl];
                    float cc[NS];
                    ld_slots<NS>(cc, s.Cp + ((ln.gl * T + tt) * p.O + o) * NSL + ln.q * NS);
#pragma unroll
                    for (int sl = 0; sl < NS; ++sl) Gv[sl] = fmaf(cc[sl], dyo, Gv[sl]);
                }
            }
            // sum_p G[n,p] u[r,p]  and  sum_n B[n,r] G[n,p] (ZOH: B^T Z^T G)
            float gw[NS];
#pragma unroll
            for (int sl = 0; sl < NS; ++sl) gw[sl] = Gv[sl];
            if (p.zoh) {
                float zz[NS];
                ld_slots<NS>(zz, s.zc + (ln.hc * T + tt) * NSL + ln.q * NS);
                zoh_apply_T<NR, NPR>(gw, zz);
            }
            float v[KV];
#pragma unroll
            for (int r = 0; r < RM; ++r) {
                const float ur = r < p.R ? s.u[((ln.hc * T + tt) * p.R + r) * PP + ln.pl] : 0.f;
                float bb[NS];
                ld_slots<NS>(bb, s.Bp + ((ln.gl * T + tt) * p.R + (r < p.R ? r : 0)) * NSL + ln.q * NS);
                float du = 0.f;
#pragma unroll
                for (int sl = 0; sl < NS; ++sl) {
                    v[r * NS + sl] = Gv[sl] * ur;
                    du = fmaf(bb[sl], gw[sl], du);
                }
                if (r < p.R) redB[(((ln.hc * T + tt) * RM + r) * NQ + ln.q) * PP + ln.pl] = du;
            }
            xreduce<KV, S>(v, lane_in_s);
            put_reduced<KV, S>(redA + (((ln.hc * T + tt) * NWP + wp) * NQ + ln.q) * KV, v,
                               lane_in_s);
            float cf[NS];
            ld_slots<NS>(cf, s.coef + (ln.hc * T + tt) * NSL + ln.q * NS);
            // G <- A_t^T G
            step_adj<NR, NPR>(Gv, cf);
        }
        __syncthreads();
        // dx_t = sigma_t sum_q(B^T G) - beta_{t+1} M^T dy + D dy
        const Lanes2D lq = lanes2d(p.P);
        for (int row = lq.ty; row < HC * T * p.R; row += lq.ny)
        for (int q = lq.tx; q < p.P; q += lq.W) {
            const int r = row % p.R, tt = (row / p.R) % T, hc = row / (p.R * T);
            int h = ln.hbase + hc, t = t0 + tt;
            if (h >= p.H || t >= p.L) continue;
            float acc = 0.f;
            for (int k = 0; k < NQ; ++k) acc += redB[(((hc * T + tt) * RM + r) * NQ + k) * PP + q];
            float v = acc * s.sig[hc * T + tt];
            const float bnx = s.bn[hc * T + tt];
            for (int o = 0; o < p.O; ++o)
                v = fmaf(-bnx * s.corr[((hc * T + tt) * p.O + o) * p.R + r],
                         s.dy[((hc * T + tt) * p.O + o) * PP + q], v);
            if (p.O == p.R) v = fmaf(p.D[h], s.dy[((hc * T + tt) * p.O + r) * PP + q], v);
            st_io(p.dx, ix_x(p, ln.b, t, h, r, q), v, p.bf16);
        }
        // gbu_t[r][n] and M2_t[o][r], corr2_t
        const Lanes2D ln2 = lanes2d(p.N);
        for (int row = ln2.ty; row < HC * T * p.R; row += ln2.ny)
        for (int n = ln2.tx; n < p.N; n += ln2.W) {
            const int r = row % p.R, tt = (row / p.R) % T, hc = row / (p.R * T);
            int h = ln.hbase + hc, t = t0 + tt;
            if (h >= p.H || t >= p.L) continue;
            int sl = s.slot[n];
            int q = sl / NS, k = r * NS + sl % NS;
            float acc = 0.f;
            for (int w2 = 0; w2 < NWP; ++w2) acc += redA[(((hc * T + tt) * NWP + w2) * NQ + q) * KV + k];
            p.ws_gbu[ix_wsk(p, ln.b, t, h, r, p.R, n)] = acc;
        }
        for (int i = threadIdx.x; i < HC * T * p.O * p.R; i += blockDim.x) {
            int r = i % p.R, o = (i / p.R) % p.O, tt = (i / (p.R * p.O)) % T,
                hc = i / (p.R * p.O * T);
            int h = ln.hbase + hc, t = t0 + tt;
            if (h >= p.H || t >= p.L) continue;
            float acc = 0.f;
            for (int q = 0; q < p.P; ++q)
                acc = fmaf(s.dy[((hc * T + tt) * p.O + o) * PP + q],
                           s.u[((hc * T + tt) * p.R + r) * PP + q], acc);
            p.ws_M2[((ix_bth(p, ln.b, t, h)) * p.O + o) * p.R + r] = acc;
        }
        __syncthreads();
        // dsigma_t = sum_{r,n} B[n,r] gbu[r][n];  corr2_t = sum_{o,r} M[o][r] M2[o][r]
        // one warp per token, lanes over (r, n), fixed-order shuffle reduction
        {
            const int wid = threadIdx.x >> 5, lid = threadIdx.x & 31, nw = blockDim.x >> 5;
            for (int i = wid; i < HC * T; i += nw) {
                const int hc = i / T, tt = i - hc * T, h = ln.hbase + hc, t = t0 + tt;
                if (h >= p.H || t >= p.L) continue;
                const int gl = h / p.hpg - ln.gbase;
                float ds = 0.f;
                for (int k = lid; k < p.R * p.N; k += 32) {
                    const int r = k / p.N, n = k - r * p.N;
                    const int sl = s.slot[n], q = sl / NS;
                    float g = 0.f;
                    for (int w2 = 0; w2 < NWP; ++w2)
                        g += redA[(((hc * T + tt) * NWP + w2) * NQ + q) * KV + r * NS + (sl - q * NS)];
                    ds = fmaf(s.Bp[((gl * T + tt) * p.R + r) * NSL + sl], g, ds);
                }
#pragma unroll
                for (int o = 16; o >= 1; o >>= 1) ds += __shfl_xor_sync(0xffffffffu, ds, o);
                if (lid == 0) {
                    float c2 = 0.f;
                    for (int o = 0; o < p.O; ++o)
                        for (int r = 0; r < p.R; ++r)
                            c2 = fmaf(s.corr[((hc * T + tt) * p.O + o) * p.R + r],
                                      p.ws_M2[((ix_bth(p, ln.b, t, h)) * p.O + o) * p.R + r], c2);
                    p.ws_tok[ix_bth(p, ln.b, t, h) * 2 + 0] = ds;
                    p.ws_tok[ix_bth(p, ln.b, t, h) * 2 + 1] = c2;
                }
            }
        }
        __syncthreads();
    }
    // after step 0: G = dL/dK_{-1};  dh0 = G, dw0 = beta_0 G, dbeta_0 = <G, w0>
    float beta0 = 0.f;
    if (ln.hv && p.two_ep && p.L > 0)
        beta0 = (1.f - ld_io(p.lam, ix_lam(p, ln.b, 0, ln.h), p.bf16)) *
                ld_io(p.dt, ix_dt(p, ln.b, 0, ln.h), p.bf16);
    float db0 = 0.f;
#pragma unroll
    for (int sl = 0; sl < NS; ++sl) {
        int n = row_of<NR, NPR>(ln.q, sl, p.nr, p.np, NQ);
        if (!act || n < 0) continue;
        long long ii = ix_st(p, ln.b, ln.h, n, ln.pl);
        if (p.dh0) p.dh0[ii] = Gv[sl];
        if (p.dw0) p.dw0[ii] = beta0 * Gv[sl];
        if (p.w0) db0 = fmaf(Gv[sl], p.w0[ii], db0);
    }
    (void)cf0;
    // block reduction of dbeta_0 per head (fixed order)
    float *rb = s.red;
    __syncthreads();
    rb[threadIdx.x] = db0;
    __syncthreads();
    if (threadIdx.x < HC) {
        int hc = threadIdx.x, h = ln.hbase + hc;
        if (h < p.H) {
            float acc = 0.f;
            for (int k = 0; k < PP * NQ; ++k) acc += rb[hc * PP * NQ + k];
            p.ws_par[((long long)ln.b * p.H + h) * npar_of(p) + p.ndec + p.np + 1] = acc;
        }
    }
}

// ------------------------------------------------------------------------
// backward finalize: decay/angle gradients by reverse cumulative sums over
// time, done as a two-level scan.  Blocks of TBL tokens run in parallel
// (k_bwd_units_local: local suffix sums, block totals), a per-(b, h) pass
// carries the totals across blocks (k_bwd_units_carry), and an elementwise
// pass writes ddt and dlambda (k_bwd_units_final).  All sums run in a fixed
// order.
// ------------------------------------------------------------------------
constexpr int FT = 32;
constexpr int TBL = 64;   // equal to the tensor-core chunk, whose boundaries carry exact values

__host__ __device__ inline int ntb_of(const Params &p) { return (p.L + TBL - 1) / TBL; }

// per-mode constants shared by the finalize kernels
struct ModeInfo {
    float a, w;
    int n0;
    bool pair, valid;
};
__device__ __forceinline__ ModeInfo mode_info(const Params &p, int h, int m) {
    ModeInfo mi;
    const int nmode = p.nr + p.np;
    mi.valid = m < nmode;
    mi.a = mi.w = 0.f;
    mi.pair = mi.valid && m >= p.nr;
    mi.n0 = 0;
    if (mi.valid) {
        mi.a = neg_exp(p.A_log[h * p.ndec + (p.per_coord ? m : 0)]);
        // per-token angles: the angle's gradient leaves through dtheta, not ddt
        if (mi.pair && !p.angle_tok) mi.w = p.theta[h * p.np + (m - p.nr)];
        mi.n0 = m < p.nr ? m : p.nr + 2 * (m - p.nr);
    }
    return mi;
}

__device__ __forceinline__ void units_local_item(const Params &p, float *smem, int tb, int h,
                                                 int b) {
    const int m = threadIdx.x, nthr = blockDim.x;
    const int g = h / p.hpg;
    const int NTB = ntb_of(p), nmode = p.nr + p.np;
    const int tbeg = tb * TBL, tend = min(p.L, tbeg + TBL);
    float *s_c = smem;  // [FT][nthr]
    const ModeInfo mi = mode_info(p, h, m);
    float cr = 0.f, ci = 0.f, dA = 0.f, dth = 0.f, dD = 0.f, sdt = 0.f;
    for (int t1 = tend; t1 > tbeg; t1 -= FT) {
        const int t0 = max(tbeg, t1 - FT), tn = t1 - t0;
        for (int k = tn - 1; k >= 0; --k) {
            const int t = t0 + k;
            const float dv = ld_io(p.dt, ix_dt(p, b, t, h), p.bf16);
            float contrib = 0.f;
            if (mi.valid) {
                const float lv = p.two_ep ? ld_io(p.lam, ix_lam(p, b, t, h), p.bf16) : 1.f;
                float bnx = 0.f;
                if (t + 1 < p.L && p.two_ep)
                    bnx = (1.f - ld_io(p.lam, ix_lam(p, b, t + 1, h), p.bf16)) *
                          ld_io(p.dt, ix_dt(p, b, t + 1, h), p.bf16);
                const float sig = lv * dv + bnx;
                const float *M2 = p.ws_M2 + ix_bth(p, b, t, h) * p.O * p.R;
                const int n0 = mi.n0;
                const bool pair = mi.pair;
                float xr = 0.f, xi = 0.f, yr = 0.f, yi = 0.f;
                for (int o = 0; o < p.O; ++o) {
                    // dCK[o][n] = dC[o][n] + beta_{t+1} sum_r B[r][n] M2[o][r]
                    float k0 = p.ws_dC[ix_wsk(p, b, t, h, o, p.O, n0)];
                    float k1 = pair ? p.ws_dC[ix_wsk(p, b, t, h, o, p.O, n0 + 1)] : 0.f;
                    for (int r = 0; r < p.R; ++r) {
                        const float mm = bnx * M2[o * p.R + r];
                        k0 = fmaf(mm, ld_io(p.Bm, ix_B(p, b, t, g, r, n0), p.bf16), k0);
                        if (pair) k1 = fmaf(mm, ld_io(p.Bm, ix_B(p, b, t, g, r, n0 + 1), p.bf16), k1);
                    }
                    const float c0 = ld_io(p.Cm, ix_C(p, b, t, g, o, n0), p.bf16);
                    const float c1 = pair ? ld_io(p.Cm, ix_C(p, b, t, g, o, n0 + 1), p.bf16) : 0.f;
                    xr += c0 * k0 + c1 * k1;   // conj(c) * k
                    xi += c0 * k1 - c1 * k0;
                }
                for (int r = 0; r < p.R; ++r) {
                    const float b0 = ld_io(p.Bm, ix_B(p, b, t, g, r, n0), p.bf16);
                    const float b1 = pair ? ld_io(p.Bm, ix_B(p, b, t, g, r, n0 + 1), p.bf16) : 0.f;
                    const float g0 = p.ws_gbu[ix_wsk(p, b, t, h, r, p.R, n0)];
                    const float g1 = pair ? p.ws_gbu[ix_wsk(p, b, t, h, r, p.R, n0 + 1)] : 0.f;
                    yr += b0 * g0 + b1 * g1;   // b * conj(g)
                    yi += b1 * g0 - b0 * g1;
                }
                float zoh_dt = 0.f, zoh_dw = 0.f;
                if (p.zoh) {
                    // the write of step t is Z b u: Y = Z b conj(g); the gradient of Z,
                    // (yr, -yi), reaches dt, a and the angle through dZ/d.
                    float phi = 0.f;
                    if (pair)
                        phi = p.angle_tok ? p.theta[ix_th(p, b, t, h, m - p.nr)]
                                          : dv * p.theta[h * p.np + (m - p.nr)];
                    float f1r, f1i, fdr, fdi;
                    zoh_phi(dv * mi.a, phi, f1r, f1i, fdr, fdi);
                    const float gzr = yr, gzi = -yi;
                    float zdr, zdi;   // dZ / d dt
                    if (pair && p.angle_tok) {
                        zdr = fmaf(dv * mi.a, fdr, f1r);
                        zdi = fmaf(dv * mi.a, fdi, f1i);
                    } else {
                        float sn, cs;
                        sincosf(phi, &sn, &cs);
                        const float ex = expf(dv * mi.a);
                        zdr = ex * cs;
                        zdi = ex * sn;
                    }
                    zoh_dt = fmaf(gzr, zdr, gzi * zdi);
                    // dZ / da = dt^2 phi1'; dZ / dangle = i dt phi1' (per token) or i dt^2 phi1'
                    dA = fmaf(dv * dv, fmaf(gzr, fdr, gzi * fdi), dA);
                    const float wsc = (pair && p.angle_tok) ? dv : dv * dv;
                    zoh_dw = wsc * fmaf(-gzr, fdi, gzi * fdr);
                    float nr_, ni_;
                    cmulf(dv * f1r, dv * f1i, yr, yi, nr_, ni_);
                    yr = nr_;
                    yi = ni_;
                } else {
                    yr *= sig;
                    yi *= sig;
                }
                cr += xr - yr;
                ci += xi - yi;
                // a static row's log-transition is a itself: weight 1, nothing to ddt
                const bool stat = m < p.nst;
                dA = fmaf(stat ? 1.f : dv, cr, dA);
                if (pair) dth = fmaf(dv, -ci, dth) + zoh_dw;
                // per-token angle: the local part of dL/dphi_t (the carry from
                // later time blocks is added by k_bwd_units_carry)
                if (pair && p.angle_tok) p.dtheta[ix_th(p, b, t, h, m - p.nr)] = zoh_dw - ci;
                contrib = stat ? 0.f : mi.a * cr + (pair ? -mi.w * ci : 0.f) + zoh_dt;
            }
            if (m == 0) {
                sdt += dv;
                if (p.O == p.R)
                    for (int o = 0; o < p.O; ++o)
                        dD += p.ws_M2[ix_bth(p, b, t, h) * p.O * p.R + o * p.R + o];
            }
            s_c[k * nthr + m] = contrib;
        }
        __syncthreads();
        if (m < tn) {
            float acc = 0.f;
            for (int j = 0; j < nthr; ++j) acc += s_c[m * nthr + j];
            p.ws_ddt[ix_bth(p, b, t0 + m, h)] = acc;
        }
        __syncthreads();
    }
    float *blk = p.ws_blk + (((long long)b * p.H + h) * NTB + tb) * (4 * (long long)nmode + 2);
    if (mi.valid) {
        blk[4 * m + 0] = cr;
        blk[4 * m + 1] = ci;
        blk[4 * m + 2] = dA;
        blk[4 * m + 3] = dth;
    }
    if (m == 0) {
        blk[4 * nmode + 0] = sdt;
        blk[4 * nmode + 1] = dD;
    }
}

// one (time block, head, batch row) item per block iteration; a capped grid
// strides over them
__global__ void __launch_bounds__(256) k_bwd_units_local(Params p) {
    if (gated_off(p)) return;
    extern __shared__ __align__(16) float smem[];
    const int NTB = ntb_of(p);
    const long long items = (long long)NTB * p.H * p.Bsz;
    for (long long it = blockIdx.x; it < items; it += gridDim.x) {
        const long long r = it / NTB;
        units_local_item(p, smem, (int)(it - r * NTB), (int)(r % p.H), (int)(r / p.H));
        __syncthreads();
    }
}

// carry the block totals across time blocks: per (b, h), one thread per mode
constexpr int CARRY_GROUP = 32;   // time blocks per group when the carries are exact

// sum over the block's threads of v[0 .. nthr) by warp 0 (lane-strided partials, then a
// shuffle tree: a fixed order); the total is valid in lane 0
__device__ __forceinline__ float sum_modes(const float *v, int nthr, int lane) {
    float acc = 0.f;
    for (int k = lane; k < nthr; k += 32) acc += v[k];
#pragma unroll
    for (int o = 16; o; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    return acc;
}

__host__ __device__ inline int carry_threads(const Params &p) {   // one per mode
    const int n = ((p.nr + p.np + 31) / 32) * 32;
    return n < 32 ? 32 : n;
}

__global__ void __launch_bounds__(1024) k_bwd_units_carry(Params p) {
    if (gated_off(p)) return;
    extern __shared__ __align__(16) float smem[];
    const int h = blockIdx.x, b = blockIdx.y;
    // thread (mode m, slice s): with exact carries the slices take interleaved time blocks
    const int nthr = carry_threads(p), nsub = blockDim.x / nthr;
    const int m = threadIdx.x % nthr, sl = threadIdx.x / nthr;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int NTB = ntb_of(p), nmode = p.nr + p.np;
    const long long bstride = 4 * (long long)nmode + 2;
    const float *blk0 = p.ws_blk + ((long long)b * p.H + h) * NTB * bstride;
    float *blkc = p.ws_blkc + ((long long)b * p.H + h) * NTB;
    const ModeInfo mi = mode_info(p, h, m);
    float *s_c = smem;  // [nthr], or [CARRY_GROUP][nthr] when the carries are exact
    float car = 0.f, cai = 0.f, dA = 0.f, dth = 0.f, dD = 0.f;
    if (p.ws_qb) {
        // The chunked chain left the exact carry at every block start (sum_p conj(Gbar) A
        // K_prev at the next block's start, four partial sums over column blocks of p), so
        // the blocks are independent: groups of CARRY_GROUP blocks, the slices forming
        // their modes' terms of interleaved blocks, then one warp per block summing the
        // modes.
        const float *q0 = p.ws_qb + ((long long)b * p.H + h) * p.nc * 4 * (long long)p.N;
        for (int g0 = NTB - 1; g0 >= 0; g0 -= CARRY_GROUP) {
            const int ng = min(CARRY_GROUP, g0 + 1);
#pragma unroll 4
            for (int j = sl; j < ng; j += nsub) {
                const int tb = g0 - j;
                const float *blk = blk0 + tb * bstride;
                float contrib = 0.f;
                if (mi.valid) {
                    float cr = 0.f, ci = 0.f;
                    if (tb + 1 < NTB) {
                        const float *q = q0 + (long long)(tb + 1) * 4 * p.N;
                        for (int w2 = 0; w2 < 4; ++w2) {
                            cr += q[w2 * p.N + mi.n0];
                            if (mi.pair) ci += q[w2 * p.N + mi.n0 + 1];
                        }
                    }
                    const bool stat = m < p.nst;
                    const float sdt = blk[4 * nmode + 0];
                    const float ntok = (float)(min(p.L, (tb + 1) * TBL) - tb * TBL);
                    dA += blk[4 * m + 2] + cr * (stat ? ntok : sdt);
                    if (mi.pair) dth += blk[4 * m + 3] - ci * sdt;
                    contrib = stat ? 0.f : mi.a * cr + (mi.pair ? -mi.w * ci : 0.f);
                }
                s_c[j * nthr + m] = contrib;
                if (m == 0) dD += blk[4 * nmode + 1];
            }
            __syncthreads();
            for (int j = warp; j < ng; j += blockDim.x >> 5) {
                const float acc = sum_modes(s_c + j * nthr, nthr, lane);
                if (lane == 0) blkc[g0 - j] = acc;
            }
            __syncthreads();
        }
        // the slices' partial sums, added in slice order
        s_c[sl * nthr + m] = dA;
        s_c[(nsub + sl) * nthr + m] = dth;
        s_c[(2 * nsub + sl) * nthr + m] = dD;
        __syncthreads();
        if (sl == 0) {
            dA = dth = dD = 0.f;
            for (int k = 0; k < nsub; ++k) {
                dA += s_c[k * nthr + m];
                dth += s_c[(nsub + k) * nthr + m];
                dD += s_c[(2 * nsub + k) * nthr + m];
            }
        }
        __syncthreads();
    } else {
        for (int tb = NTB - 1; tb >= 0; --tb) {
            const float *blk = blk0 + tb * bstride;
            const float sdt = blk[4 * nmode + 0];
            float contrib = 0.f;
            if (mi.valid) {
                const bool stat = m < p.nst;
                // static rows: the carried sum counts once per token of the block
                const float ntok = (float)(min(p.L, (tb + 1) * TBL) - tb * TBL);
                dA += blk[4 * m + 2] + car * (stat ? ntok : sdt);
                if (mi.pair) dth += blk[4 * m + 3] - cai * sdt;
                contrib = stat ? 0.f : mi.a * car + (mi.pair ? -mi.w * cai : 0.f);
                // per-token angles: the angle's gradient takes the carry at every token
                if (mi.pair && p.angle_tok && cai != 0.f) {
                    const int tend = min(p.L, (tb + 1) * TBL);
                    for (int t = tb * TBL; t < tend; ++t)
                        p.dtheta[ix_th(p, b, t, h, m - p.nr)] -= cai;
                }
            }
            s_c[m] = contrib;
            __syncthreads();
            if (warp == 0) {
                const float acc = sum_modes(s_c, nthr, lane);
                if (lane == 0) {
                    blkc[tb] = acc;
                    dD += blk[4 * nmode + 1];
                }
            }
            if (mi.valid) {
                car += blk[4 * m + 0];
                cai += blk[4 * m + 1];
            }
            __syncthreads();
        }
    }
    float *part = p.ws_par + ((long long)b * p.H + h) * npar_of(p);
    if (sl == 0) s_c[m] = dA;
    __syncthreads();
    if (sl != 0) return;
    if (p.per_coord) {
        if (mi.valid) part[m] = dA;
    } else if (m == 0) {
        float acc = 0.f;
        for (int j = 0; j < nmode; ++j) acc += s_c[j];
        part[0] = acc;
    }
    if (mi.pair && !p.angle_tok) part[p.ndec + (m - p.nr)] = dth;
    if (m == 0) part[p.ndec + p.np] = dD;
}

// ddt and dlambda per (b, t, h)
__global__ void k_bwd_units_final(Params p) {
    if (gated_off(p)) return;
    const long long total = (long long)p.Bsz * p.L * p.H;
    const int NTB = ntb_of(p);
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
         i += (long long)gridDim.x * blockDim.x) {
        const int h = (int)(i % p.H);
        const long long bt = i / p.H;
        const int t = (int)(bt % p.L), b = (int)(bt / p.L);
        const float dv = ld_io(p.dt, ix_dt(p, b, t, h), p.bf16);
        const float lv = p.two_ep ? ld_io(p.lam, ix_lam(p, b, t, h), p.bf16) : 1.f;
        const float ds = p.ws_tok[i * 2 + 0];
        float dd = p.ws_ddt[i] + p.ws_blkc[((long long)b * p.H + h) * NTB + t / TBL];
        if (p.two_ep) {
            // dgamma_t = dsigma_t ; dbeta_t = dsigma_{t-1} - corr2_{t-1} (t >= 1)
            float dbeta;
            if (t >= 1)
                dbeta = p.ws_tok[ix_bth(p, b, t - 1, h) * 2 + 0] -
                        p.ws_tok[ix_bth(p, b, t - 1, h) * 2 + 1];
            else
                dbeta = p.ws_par[((long long)b * p.H + h) * npar_of(p) + p.ndec + p.np + 1];
            dd += lv * ds + (1.f - lv) * dbeta;
            if (p.dlam) st_io(p.dlam, ix_lam(p, b, t, h), dv * (ds - dbeta), p.bf16);
        } else if (!p.zoh) {   // the ZOH write's dt-dependence is in ws_ddt already
            dd += ds;
        }
        st_io(p.ddt, ix_dt(p, b, t, h), dd, p.bf16);
    }
}

// (Z^T gbu)[n] of head h at step t under the ZOH write: gbu scaled by the
// mode's Z (transposed complex product on a pair)
__device__ __forceinline__ float zoh_gbu(const Params &p, int b, int t, int h, int r, int n) {
    const float dv = ld_io(p.dt, ix_dt(p, b, t, h), p.bf16);
    const bool pair = n >= p.nr;
    const int m = pair ? p.nr + (n - p.nr) / 2 : n;
    const float a = neg_exp(p.A_log[h * p.ndec + (p.per_coord ? m : 0)]);
    float phi = 0.f;
    if (pair)
        phi = p.angle_tok ? p.theta[ix_th(p, b, t, h, m - p.nr)] : dv * p.theta[h * p.np + (m - p.nr)];
    float f1r, f1i, fdr, fdi;
    zoh_phi(dv * a, phi, f1r, f1i, fdr, fdi);
    const float zr = dv * f1r, zi = dv * f1i;
    if (!pair) return zr * p.ws_gbu[ix_wsk(p, b, t, h, r, p.R, n)];
    const int n0 = p.nr + 2 * (m - p.nr);
    const float gr = p.ws_gbu[ix_wsk(p, b, t, h, r, p.R, n0)];
    const float gi = p.ws_gbu[ix_wsk(p, b, t, h, r, p.R, n0 + 1)];
    return n == n0 ? fmaf(zr, gr, zi * gi) : fmaf(-zi, gr, zr * gi);
}

// dB, dC per (b, t): sum over the heads of each group; per-head scalars first
__device__ __forceinline__ void groups_item(const Params &p, float *smem, int t, int b) {
    float *s_sig = smem, *s_bn = smem + p.H;
    for (int h = threadIdx.x; h < p.H; h += blockDim.x) {
        const float dv = ld_io(p.dt, ix_dt(p, b, t, h), p.bf16);
        const float lv = p.two_ep ? ld_io(p.lam, ix_lam(p, b, t, h), p.bf16) : 1.f;
        float bnx = 0.f;
        if (t + 1 < p.L && p.two_ep)
            bnx = (1.f - ld_io(p.lam, ix_lam(p, b, t + 1, h), p.bf16)) *
                  ld_io(p.dt, ix_dt(p, b, t + 1, h), p.bf16);
        s_sig[h] = lv * dv + bnx;
        s_bn[h] = bnx;
    }
    __syncthreads();
    const Lanes2D l = lanes2d(p.N);
    for (int row = l.ty; row < p.G * (p.R + p.O); row += l.ny) {
        const int k = row % (p.R + p.O), g = row / (p.R + p.O);
        for (int n = l.tx; n < p.N; n += l.W) {
            float acc = 0.f;
            if (k < p.R) {
                const int r = k;
                for (int h = g * p.hpg; h < (g + 1) * p.hpg; ++h) {
                    float v;
                    if (p.zoh) {
                        v = zoh_gbu(p, b, t, h, r, n);
                    } else {
                        v = s_sig[h] * p.ws_gbu[ix_wsk(p, b, t, h, r, p.R, n)];
                    }
                    const float bnx = s_bn[h];
                    if (bnx != 0.f) {
                        const float *M2 = p.ws_M2 + ix_bth(p, b, t, h) * p.O * p.R;
                        for (int o = 0; o < p.O; ++o)
                            v = fmaf(-bnx * ld_io(p.Cm, ix_C(p, b, t, g, o, n), p.bf16),
                                     M2[o * p.R + r], v);
                    }
                    acc += v;
                }
                st_io(p.dBm, ix_B(p, b, t, g, r, n), acc, p.bf16);
            } else {
                const int o = k - p.R;
                for (int h = g * p.hpg; h < (g + 1) * p.hpg; ++h)
                    acc += p.ws_dC[ix_wsk(p, b, t, h, o, p.O, n)];
                st_io(p.dCm, ix_C(p, b, t, g, o, n), acc, p.bf16);
            }
        }
    }
}

// one (token, batch row) item per block iteration; a capped grid strides over them
__global__ void __launch_bounds__(256) k_bwd_groups(Params p) {
    if (gated_off(p)) return;
    extern __shared__ __align__(16) float smem[];
    const long long items = (long long)p.L * p.Bsz;
    for (long long it = blockIdx.x; it < items; it += gridDim.x) {
        groups_item(p, smem, (int)(it % p.L), (int)(it / p.L));
        __syncthreads();
    }
}

// parameter gradients: sum the per-unit partials over the batch
__global__ void k_bwd_params(Params p) {
    if (gated_off(p)) return;
    const int np1 = npar_of(p);
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < p.H * (p.ndec + p.np + 1);
         i += gridDim.x * blockDim.x) {
        int h = i / (p.ndec + p.np + 1), k = i % (p.ndec + p.np + 1);
        float acc = 0.f;
        for (int b = 0; b < p.Bsz; ++b) acc += p.ws_par[((long long)b * p.H + h) * np1 + k];
        if (k < p.ndec) {
            p.dA_log[h * p.ndec + k] = acc * neg_exp(p.A_log[h * p.ndec + k]);
        } else if (k < p.ndec + p.np) {
            if (p.dtheta && !p.angle_tok) p.dtheta[h * p.np + (k - p.ndec)] = acc;
        } else if (p.dD) {
            p.dD[h] = (p.O == p.R) ? acc : 0.f;
        }
    }
}

// L == 0: hT = h0, last_write = prev_write (zeros if absent)
__global__ void k_copy_state(Params p) {
    long long total = (long long)p.Bsz * p.H * p.N * p.P;
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
         i += (long long)gridDim.x * blockDim.x) {
        if (p.hT) p.hT[i] = p.h0 ? p.h0[i] : 0.f;
        if (p.wT) p.wT[i] = p.w0 ? p.w0[i] : 0.f;
    }
}

// ------------------------------------------------------------------------
// host side: geometry and launches
// ------------------------------------------------------------------------
struct Combo {
    int NR, NPR;
};
static const Combo kCombos[] = {{16, 8}, {32, 0}, {8, 4}, {16, 0}, {0, 16}};

static int pick_combo(const Params &p, int &NQ) {
    int best = -1, bestw = 1 << 30, bestq = 0;
    for (int c = 0; c < 5; ++c) {
        const Combo &k = kCombos[c];
        if (p.np > 0 && k.NPR == 0) continue;
        if (p.nr > 0 && k.NR == 0) continue;
        int q1 = k.NR ? (p.nr + k.NR - 1) / k.NR : 0;
        int q2 = k.NPR ? (p.np + k.NPR - 1) / k.NPR : 0;
        int q = q1 > q2 ? q1 : q2;
        if (q < 1) q = 1;
        int waste = q * (k.NR + 2 * k.NPR) - p.N;
        if (waste < bestw) {
            bestw = waste;
            best = c;
            bestq = q;
        }
    }
    NQ = bestq;
    return best;
}

enum KernelKind { KK_FWD = 0, KK_S1 = 1, KK_S2 = 2 };

static size_t red_floats(const Params &p, int kind, int NS, int RM) {
    const Geometry &g = p.geo;
    const int NWP = g.PP > 32 ? g.PP / 32 : 1;
    if (kind == KK_FWD) return (size_t)g.HC * g.T * p.O * g.NQ * g.PP;
    size_t a = (size_t)g.HC * g.T * NWP * g.NQ * RM * NS;
    if (kind == KK_S1) return a;
    size_t bsz = (size_t)g.HC * g.T * RM * g.NQ * g.PP;
    size_t s = a + bsz;
    size_t nthr = (size_t)g.PP * g.NQ * g.HC;
    return s > nthr ? s : nthr;
}

// Choose PP, NQ, HC, T for one kernel kind; returns smem bytes (0 if impossible).
static size_t plan(Params &p, int kind, int &combo, int &RM, int &S) {
    Geometry &g = p.geo;
    int NQ;
    combo = pick_combo(p, NQ);
    if (combo < 0) return 0;
    const Combo &k = kCombos[combo];
    const int NS = k.NR + 2 * k.NPR;
    RM = (p.R <= 1 && p.O <= 1) ? 1 : 4;
    g.PP = p.P == 1 ? 1 : (p.P <= 16 ? 16 : (p.P <= 32 ? 32 : (p.P <= 64 ? 64 : 128)));
    S = g.PP == 1 ? 1 : (g.PP == 16 ? 16 : 32);
    g.NQ = NQ;
    int per_head = g.PP * NQ;
    if (per_head > MAXT) return 0;
    int hc = MAXT / per_head;
    if (hc > 64) hc = 64;
    if (hc > p.H) hc = p.H;
    if (hc < 1) hc = 1;
    // whole warps: full-mask shuffles need every lane present
    while ((per_head * hc) % 32 != 0 && per_head * (hc + 1) <= MAXT) ++hc;
    if ((per_head * hc) % 32 != 0 && S > 1) return 0;
    g.HC = hc;
    const int NSL = NQ * NS;
    int ngl = (hc - 1) / p.hpg + 2;
    if (ngl > hc) ngl = hc;
    for (int T = 32; T >= 1; T /= 2) {
        g.T = T;
        size_t fl = smem_floats(p, NSL, ngl, red_floats(p, kind, NS, RM), kind != KK_FWD);
        if (fl * 4 <= 160 * 1024) return fl * 4;
    }
    return 0;
}

template <int NR, int NPR>
constexpr int combo_id() {
    return NR == 16 && NPR == 8 ? 0 : (NR == 32 ? 1 : (NR == 8 ? 2 : (NR == 16 ? 3 : 4)));
}

template <int NR, int NPR, int RM, int S>
static cudaError_t launch_kind(int kind, const Params &p, dim3 grid, dim3 block, size_t sm,
                               cudaStream_t st) {
    if (kind == KK_FWD) {
        auto fn = k_fwd<NR, NPR, RM>;
        cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
        fn<<<grid, block, sm, st>>>(p);
        profile_mark(st, "k_fwd");
    } else if (kind == KK_S1) {
        auto fn = k_bwd_sweep1<NR, NPR, RM, S>;
        cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
        fn<<<grid, block, sm, st>>>(p);
        profile_mark(st, "k_bwd_sweep1");
    } else {
        auto fn = k_bwd_sweep2<NR, NPR, RM, S>;
        cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
        fn<<<grid, block, sm, st>>>(p);
        profile_mark(st, "k_bwd_sweep2");
    }
    return cudaGetLastError();
}

#define SSM_CASE1(NR, NPR, RM, S)                                                                \
    case combo_id<NR, NPR>() * 100 + RM * 10 + S:                                               \
        return launch_kind<NR, NPR, RM, S>(kind, p, grid, block, sm, st);
#define SSM_CASES(NR, NPR)                                                                       \
    SSM_CASE1(NR, NPR, 1, 1)                                                                     \
    SSM_CASE1(NR, NPR, 1, 16) SSM_CASE1(NR, NPR, 1, 32) SSM_CASE1(NR, NPR, 4, 1)                 \
        SSM_CASE1(NR, NPR, 4, 16) SSM_CASE1(NR, NPR, 4, 32)

static cudaError_t launch_scan(int kind, Params p, cudaStream_t st) {
    int combo, RM, S;
    size_t sm = plan(p, kind, combo, RM, S);
    if (sm == 0) return cudaErrorInvalidConfiguration;
    const Geometry &g = p.geo;
    dim3 grid((p.H + g.HC - 1) / g.HC, p.Bsz);
    dim3 block(g.PP * g.NQ * g.HC);
    switch (combo * 100 + RM * 10 + S) {
        SSM_CASES(16, 8)
        SSM_CASES(32, 0)
        SSM_CASES(8, 4)
        SSM_CASES(16, 0)
        SSM_CASES(0, 16)
        default:
            return cudaErrorInvalidConfiguration;
    }
}

// Whether the SIMT path supports these sizes (host check before launching).
bool simt_supported(const Params &p0) {
    Params p = p0;
    if (p.R > 4 || p.O > 4 || p.P > 128) return false;
    for (int kind = 0; kind < 3; ++kind) {
        int combo, RM, S;
        if (plan(p, kind, combo, RM, S) == 0) return false;
    }
    return true;
}

cudaError_t simt_forward(const Params &p, cudaStream_t st) {
    if (p.L == 0) {
        k_copy_state<<<64, 256, 0, st>>>(p);
        profile_mark(st, "k_copy_state");
        return cudaGetLastError();
    }
    return launch_scan(KK_FWD, p, st);
}

bool chunk_bwd_supported(const Params &p);
cudaError_t chunk_bwd_states(const Params &p, cudaStream_t st);
cudaError_t chunk_bwd_reverse(const Params &p, cudaStream_t st);

// Finalize passes shared by both backward chains: within-block decay sums
// (when the chain has not produced them), block carries, per-token ddt and
// dlambda, group sums of dB / dC (when the chain has not written them), and
// the batch sums of the parameter gradients.  Item grids are capped and
// strided so that a gated-off chain costs one short launch per kernel.
static cudaError_t bwd_finalize(const Params &p, cudaStream_t st, bool local, bool groups) {
    cudaError_t e;
    int nthr = ((p.nr + p.np + 31) / 32) * 32;
    if (nthr < 32) nthr = 32;
    const long long cap = 148LL * 16;
    if (local) {
        const long long items = (long long)ntb_of(p) * p.H * p.Bsz;
        const int blocks = (int)(items < cap ? items : cap);
        k_bwd_units_local<<<blocks, nthr, (size_t)FT * nthr * 4, st>>>(p);
        profile_mark(st, "k_bwd_units_local");
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    {
        // with exact carries, up to four slices of the modes' threads take interleaved blocks
        const int cthr = carry_threads(p);
        const int nsub = p.ws_qb ? (1024 / cthr < 4 ? 1024 / cthr : 4) : 1;
        k_bwd_units_carry<<<dim3(p.H, p.Bsz), cthr * nsub,
                            (size_t)(p.ws_qb ? CARRY_GROUP : 1) * cthr * 4, st>>>(p);
    }
    profile_mark(st, "k_bwd_units_carry");
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const long long total = (long long)p.Bsz * p.L * p.H;
    int blocks = (int)((total + 255) / 256);
    if (blocks > 148 * 32) blocks = 148 * 32;
    k_bwd_units_final<<<blocks, 256, 0, st>>>(p);
    profile_mark(st, "k_bwd_units_final");
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if (groups) {
        const long long items = (long long)p.L * p.Bsz;
        const int gb = (int)(items < cap ? items : cap);
        k_bwd_groups<<<gb, 256, (size_t)2 * p.H * 4, st>>>(p);
        profile_mark(st, "k_bwd_groups");
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    k_bwd_params<<<4, 256, 0, st>>>(p);
    profile_mark(st, "k_bwd_params");
    return cudaGetLastError();
}

// Recurrent backward: both sweeps token by token, then the finalize passes.
cudaError_t simt_backward(const Params &p, cudaStream_t st) {
    cudaError_t e;
    if ((e = launch_scan(KK_S1, p, st)) != cudaSuccess) return e;
    if ((e = launch_scan(KK_S2, p, st)) != cudaSuccess) return e;
    return bwd_finalize(p, st, true, true);
}

// Tensor-core backward: the chunk states (unless the forward's are given), the
// chunk-parallel kernels, which also produce the within-block decay sums (and
// dB / dC when every group has one head), then the shared finalize passes.
cudaError_t chunk_backward(const Params &p, cudaStream_t st) {
    cudaError_t e;
    if ((e = chunk_bwd_states(p, st)) != cudaSuccess) return e;
    if ((e = chunk_bwd_reverse(p, st)) != cudaSuccess) return e;
    return bwd_finalize(p, st, false, p.hpg != 1);
}

}  // namespace ssm
