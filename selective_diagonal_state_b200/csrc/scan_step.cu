// One recurrent step of the selective diagonal scan (autoregressive decoding).
//
// A state-space layer run as a recurrence keeps a constant-size state per
// token at inference ("State Space Models", robocikowo.com: glossary item 2,
// the discretised recurrence x_k = A_bar x_{k-1} + B_bar u_k, y_k = C x_k, and
// the complexity entry, O(1) memory per token in autoregressive inference).
// For the recurrence of this library (two-endpoint write, real rows and 2x2
// decay-rotation pairs, rank-R routing):
//     H_t = A_t (H_{t-1} + beta_t W_{t-1}) + gamma_t W_t,   W_t = B_t u_t
//     y_t = C_t H_t + D u_t
// with A_t = e^{dt a} on a real row and e^{dt a_j} R(dt theta_j) on pair j.
// Thread (batch row, head, channel q) walks every state row of its channel, so
// the state in HBM is read and written once, coalesced over q; the transition
// of each mode is recomputed by the P threads of a head (a few special-function
// operations per row, far below the memory time).
#include "common.cuh"

namespace ssm {

namespace stepk {
constexpr int THREADS = 128;
constexpr int MAXR = 8;   // rank_in / rank_out handled by the step kernel
}  // namespace stepk

__global__ void __launch_bounds__(stepk::THREADS) k_scan_step(Params p, float *hs, float *ws) {
    const long long units = (long long)p.Bsz * p.H * p.P;
    for (long long u = blockIdx.x * (long long)blockDim.x + threadIdx.x; u < units;
         u += (long long)gridDim.x * blockDim.x) {
        const int q = (int)(u % p.P);
        const long long bh = u / p.P;
        const int h = (int)(bh % p.H), b = (int)(bh / p.H);
        const int g = h / p.hpg;
        const float dt = ld_io(p.dt, ix_dt(p, b, 0, h), p.bf16);
        const float lam = p.two_ep ? ld_io(p.lam, ix_lam(p, b, 0, h), p.bf16) : 1.f;
        const float gam = lam * dt, beta = (1.f - lam) * dt;
        float uv[stepk::MAXR], yacc[stepk::MAXR];
#pragma unroll
        for (int r = 0; r < stepk::MAXR; ++r) {
            uv[r] = r < p.R ? ld_io(p.x, ix_x(p, b, 0, h, r, q), p.bf16) : 0.f;
            yacc[r] = 0.f;
        }
        // W_t of row n = sum_r B_t[n][r] u_t[r]
        auto write_of = [&](int n) {
            float s = 0.f;
            for (int r = 0; r < p.R; ++r) s = fmaf(ld_io(p.Bm, ix_B(p, b, 0, g, r, n), p.bf16), uv[r], s);
            return s;
        };
        auto readout = [&](int n, float v) {
            for (int o = 0; o < p.O; ++o)
                yacc[o] = fmaf(ld_io(p.Cm, ix_C(p, b, 0, g, o, n), p.bf16), v, yacc[o]);
        };
        for (int n = 0; n < p.nr; ++n) {
            const float a = -expf(p.A_log[h * p.ndec + (p.per_coord ? n : 0)]);
            const float e = expf(n < p.nst ? a : dt * a);   // static rows: e^{a}
            const long long i0 = ix_st(p, b, h, n, q);
            const float wn = write_of(n);
            const float wp = (p.two_ep && ws) ? ws[i0] : 0.f;
            float wsc = gam;   // the write's scale: dt (Euler) or (e^{dt a} - 1) / a (ZOH)
            if (p.zoh) {
                float f1r, f1i, fdr, fdi;
                zoh_phi(dt * a, 0.f, f1r, f1i, fdr, fdi);
                wsc = dt * f1r;
            }
            const float hn = fmaf(e, fmaf(beta, wp, hs[i0]), wsc * wn);
            hs[i0] = hn;
            if (ws) ws[i0] = wn;
            readout(n, hn);
        }
        for (int j = 0; j < p.np; ++j) {
            const int n0 = p.nr + 2 * j;
            const float a = -expf(p.A_log[h * p.ndec + (p.per_coord ? p.nr + j : 0)]);
            const float mag = expf(dt * a);
            float sn, cs;
            // per-token angles: theta holds this token's [B][H][np] angles
            sincosf(p.angle_tok ? p.theta[((long long)b * p.H + h) * p.np + j]
                                : dt * p.theta[h * p.np + j],
                    &sn, &cs);
            const float er = mag * cs, ei = mag * sn;
            const long long i0 = ix_st(p, b, h, n0, q), i1 = ix_st(p, b, h, n0 + 1, q);
            const float wr = write_of(n0), wi = write_of(n0 + 1);
            float zr = hs[i0], zi = hs[i1];
            if (p.two_ep && ws) {
                zr = fmaf(beta, ws[i0], zr);
                zi = fmaf(beta, ws[i1], zi);
            }
            // (er + i ei)(zr + i zi) + gamma W  (ZOH: + Z W, complex)
            float ur = gam * wr, ui = gam * wi;
            if (p.zoh) {
                float f1r, f1i, fdr, fdi;
                const float phi = p.angle_tok ? p.theta[((long long)b * p.H + h) * p.np + j]
                                              : dt * p.theta[h * p.np + j];
                zoh_phi(dt * a, phi, f1r, f1i, fdr, fdi);
                ur = dt * (f1r * wr - f1i * wi);
                ui = dt * (f1i * wr + f1r * wi);
            }
            const float hr = fmaf(er, zr, fmaf(-ei, zi, ur));
            const float hi = fmaf(er, zi, fmaf(ei, zr, ui));
            hs[i0] = hr;
            hs[i1] = hi;
            if (ws) {
                ws[i0] = wr;
                ws[i1] = wi;
            }
            readout(n0, hr);
            readout(n0 + 1, hi);
        }
        for (int o = 0; o < p.O; ++o) {
            const float dterm = p.R == p.O ? p.D[h] * uv[o] : 0.f;
            st_io(p.y, ix_y(p, b, 0, h, o, q), yacc[o] + dterm, p.bf16);
        }
    }
}

bool step_supported(const Params &p) { return p.R <= stepk::MAXR && p.O <= stepk::MAXR; }

cudaError_t scan_step(const Params &p, float *h, float *w, cudaStream_t st) {
    const long long units = (long long)p.Bsz * p.H * p.P;
    long long blocks = (units + stepk::THREADS - 1) / stepk::THREADS;
    if (blocks > 148 * 16) blocks = 148 * 16;
    if (blocks < 1) blocks = 1;
    k_scan_step<<<(int)blocks, stepk::THREADS, 0, st>>>(p, h, w);
    profile_mark(st, "k_scan_step");
    return cudaGetLastError();
}

}  // namespace ssm
