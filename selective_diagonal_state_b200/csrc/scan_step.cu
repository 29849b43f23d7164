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
// the state in HBM is read and written once, coalesced over q.  The staged
// kernel computes each (batch row, head)'s transitions, write scales and B / C
// rows once per CTA in shared memory; the plain kernel (every head too wide for
// that) recomputes them in each of the head's P threads.
#include "common.cuh"

namespace ssm {

namespace stepk {
constexpr int THREADS = 128;
constexpr int MAXR = 8;   // rank_in / rank_out handled by the step kernel
constexpr size_t STAGED_SMEM_MAX = 96 * 1024;
// floats per (batch row, head) of the staged kernel: per state row two
// coefficients (a real row: its decay and write scale; a pair: (er, ei) of its
// transition on the re row, the (complex) write scale on the im row), the rows' B
// (R ranks) and C (O ranks), and beta; odd, so that lanes of different heads
// read different banks
__host__ __device__ inline int staged_floats(const Params &p) {
    return p.N * (2 + p.R + p.O) + 1;
}
// (batch row, head) pairs one CTA of the staged kernel can touch
__host__ __device__ inline int staged_bh(const Params &p) { return (THREADS + p.P - 1) / p.P + 1; }
}  // namespace stepk

// The step with the transition and write coefficients of each (batch row, head)
// computed once per CTA into shared memory (not once per channel): the P threads
// of a head then only stream the state, eight rows at a time with every load of a
// block issued before its arithmetic.  Thread = (batch row, head, channel q).
__global__ void __launch_bounds__(stepk::THREADS)
    k_scan_step_staged(Params p, float *__restrict__ hs, float *__restrict__ ws) {
    extern __shared__ float ssm_step_smem[];
    float *sm = ssm_step_smem;
    const int tid = threadIdx.x;
    const long long units = (long long)p.Bsz * p.H * p.P;
    const long long u0 = (long long)blockIdx.x * stepk::THREADS;
    const long long ulast = (u0 + stepk::THREADS < units ? u0 + stepk::THREADS : units) - 1;
    const long long bh0 = u0 / p.P;
    const int nbh = (int)(ulast / p.P - bh0 + 1);
    const int PB = stepk::staged_floats(p), N = p.N;
    // (batch row, head) of each of the CTA's pairs, once (64-bit divisions are slow)
    int *s_b = reinterpret_cast<int *>(sm + (size_t)stepk::staged_bh(p) * PB);
    int *s_h = s_b + stepk::staged_bh(p);
    for (int k = tid; k < nbh; k += stepk::THREADS) {
        const long long bh = bh0 + k;
        s_h[k] = (int)(bh % p.H);
        s_b[k] = (int)(bh / p.H);
    }
    __syncthreads();
    // ---- coefficients of the CTA's (batch row, head) pairs
    for (int i = tid; i < nbh * N; i += stepk::THREADS) {
        const int k = i / N, n = i - k * N;
        const int h = s_h[k], b = s_b[k];
        float *co = sm + k * PB;
        const float dt = ld_io(p.dt, ix_dt(p, b, 0, h), p.bf16);
        const float lam = p.two_ep ? ld_io(p.lam, ix_lam(p, b, 0, h), p.bf16) : 1.f;
        const float gam = lam * dt;
        if (n == 0) co[PB - 1] = (1.f - lam) * dt;   // beta
        if (n < p.nr) {
            const float a = -expf(p.A_log[h * p.ndec + (p.per_coord ? n : 0)]);
            float wsc = gam;   // the write's scale: dt (Euler) or (e^{dt a} - 1) / a (ZOH)
            if (p.zoh) {
                float f1, fd;
                zoh_phi_real(dt * a, f1, fd);
                wsc = dt * f1;
            }
            co[2 * n] = expf(n < p.nst ? a : dt * a);   // static rows: e^{a}
            co[2 * n + 1] = wsc;
        } else if (((n - p.nr) & 1) == 0) {
            const int j = (n - p.nr) >> 1;
            const float a = -expf(p.A_log[h * p.ndec + (p.per_coord ? p.nr + j : 0)]);
            const float mag = expf(dt * a);
            // per-token angles: theta holds this token's [B][H][np] angles
            const float phi = p.angle_tok ? p.theta[((long long)b * p.H + h) * p.np + j]
                                          : dt * p.theta[h * p.np + j];
            float sn, cs;
            sincosf(phi, &sn, &cs);
            co[2 * n] = mag * cs;
            co[2 * n + 1] = mag * sn;
            float zr = gam, zi = 0.f;   // ZOH: Z = dt phi1(dt a + i phi)
            if (p.zoh) {
                float f1r, f1i, fdr, fdi;
                zoh_phi(dt * a, phi, f1r, f1i, fdr, fdi);
                zr = dt * f1r;
                zi = dt * f1i;
            }
            co[2 * n + 2] = zr;
            co[2 * n + 3] = zi;
        }
    }
    const int RO = p.R + p.O;
    for (int i = tid; i < nbh * RO * N; i += stepk::THREADS) {
        const int k = i / (RO * N), rem = i - k * RO * N, rk = rem / N, n = rem - rk * N;
        const int h = s_h[k], b = s_b[k], g = h / p.hpg;
        const float v = rk < p.R ? ld_io(p.Bm, ix_B(p, b, 0, g, rk, n), p.bf16)
                                 : ld_io(p.Cm, ix_C(p, b, 0, g, rk - p.R, n), p.bf16);
        sm[k * PB + 2 * N + rk * N + n] = v;
    }
    __syncthreads();
    const long long u = u0 + tid;
    if (u >= units) return;   // no barrier below
    // this thread's pair and channel: u = (bh0 + k) P + q, k < nbh
    const int off = (int)(u - bh0 * p.P), k = off / p.P, q = off - k * p.P;
    const int h = s_h[k], b = s_b[k];
    const float *co = sm + (size_t)k * PB, *Bv = co + 2 * N, *Cv = Bv + p.R * N;
    const float beta = co[PB - 1];
    const bool use_w = p.two_ep && ws;
    float uv[stepk::MAXR], yacc[stepk::MAXR];
#pragma unroll
    for (int r = 0; r < stepk::MAXR; ++r) {
        uv[r] = r < p.R ? ld_io(p.x, ix_x(p, b, 0, h, r, q), p.bf16) : 0.f;
        yacc[r] = 0.f;
    }
    const long long st0 = ix_st(p, b, h, 0, q);   // row n at st0 + n * P
    const long long P = p.P;
    auto readout = [&](int n, float v) {
        for (int o = 0; o < p.O; ++o) yacc[o] = fmaf(Cv[o * N + n], v, yacc[o]);
    };
    auto write_of = [&](int n) {   // W_t of row n = sum_r B_t[n][r] u_t[r]
        float s = 0.f;
        for (int r = 0; r < p.R; ++r) s = fmaf(Bv[r * N + n], uv[r], s);
        return s;
    };
    constexpr int RB = 8;
    for (int n0 = 0; n0 < p.nr; n0 += RB) {   // real rows
        float hv[RB], wv[RB];
#pragma unroll
        for (int k = 0; k < RB; ++k) {
            const bool in = n0 + k < p.nr;
            hv[k] = in ? hs[st0 + (n0 + k) * P] : 0.f;
            wv[k] = in && use_w ? ws[st0 + (n0 + k) * P] : 0.f;
        }
#pragma unroll
        for (int k = 0; k < RB; ++k) {
            const int n = n0 + k;
            if (n >= p.nr) break;
            const float wn = write_of(n);
            const float hn = fmaf(co[2 * n], fmaf(beta, wv[k], hv[k]), co[2 * n + 1] * wn);
            hs[st0 + n * P] = hn;
            if (ws) ws[st0 + n * P] = wn;
            readout(n, hn);
        }
    }
    constexpr int PBK = RB / 2;   // pairs per block
    for (int j0 = 0; j0 < p.np; j0 += PBK) {   // rotation pairs: (re, im) rows nr + 2j, + 1
        float hv[RB], wv[RB];
#pragma unroll
        for (int k = 0; k < RB; ++k) {
            const bool in = j0 + (k >> 1) < p.np;
            const long long i = st0 + (p.nr + 2 * j0 + k) * P;
            hv[k] = in ? hs[i] : 0.f;
            wv[k] = in && use_w ? ws[i] : 0.f;
        }
#pragma unroll
        for (int jj = 0; jj < PBK; ++jj) {
            if (j0 + jj >= p.np) break;
            const int n = p.nr + 2 * (j0 + jj);
            const float er = co[2 * n], ei = co[2 * n + 1], sr = co[2 * n + 2], si = co[2 * n + 3];
            const float wr = write_of(n), wi = write_of(n + 1);
            const float zr = fmaf(beta, wv[2 * jj], hv[2 * jj]);
            const float zi = fmaf(beta, wv[2 * jj + 1], hv[2 * jj + 1]);
            // (er + i ei)(zr + i zi) + (sr + i si)(wr + i wi)
            const float hr = fmaf(er, zr, fmaf(-ei, zi, fmaf(sr, wr, -si * wi)));
            const float hi = fmaf(er, zi, fmaf(ei, zr, fmaf(sr, wi, si * wr)));
            hs[st0 + n * P] = hr;
            hs[st0 + (n + 1) * P] = hi;
            if (ws) {
                ws[st0 + n * P] = wr;
                ws[st0 + (n + 1) * P] = wi;
            }
            readout(n, hr);
            readout(n + 1, hi);
        }
    }
    for (int o = 0; o < p.O; ++o) {
        const float dterm = p.R == p.O ? p.D[h] * uv[o] : 0.f;
        st_io(p.y, ix_y(p, b, 0, h, o, q), yacc[o] + dterm, p.bf16);
    }
}

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
    if (units == 0) return cudaSuccess;
    const size_t smem = (size_t)stepk::staged_bh(p) * (stepk::staged_floats(p) + 2) * sizeof(float);
    if (smem <= stepk::STAGED_SMEM_MAX && p.P >= 16) {
        // the per-(row, head) coefficients fit in shared memory and each head has
        // enough channels to share them: the staged kernel (a head of one or a few
        // channels computes its own coefficients as cheaply as it would stage them)
        static bool done[64] = {};
        int dev = 0;
        cudaError_t e = cudaGetDevice(&dev);
        if (e != cudaSuccess) return e;
        if (smem > 48 * 1024 && !(dev >= 0 && dev < 64 && done[dev])) {
            e = cudaFuncSetAttribute(k_scan_step_staged, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)stepk::STAGED_SMEM_MAX);
            if (e != cudaSuccess) return e;
            if (dev >= 0 && dev < 64) done[dev] = true;
        }
        const long long blocks = (units + stepk::THREADS - 1) / stepk::THREADS;
        if (blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
        k_scan_step_staged<<<(int)blocks, stepk::THREADS, smem, st>>>(p, h, w);
        profile_mark(st, "k_scan_step_staged");
        return cudaGetLastError();
    }
    long long blocks = (units + stepk::THREADS - 1) / stepk::THREADS;
    if (blocks > 148 * 16) blocks = 148 * 16;
    if (blocks < 1) blocks = 1;
    k_scan_step<<<(int)blocks, stepk::THREADS, 0, st>>>(p, h, w);
    profile_mark(st, "k_scan_step");
    return cudaGetLastError();
}

}  // namespace ssm
