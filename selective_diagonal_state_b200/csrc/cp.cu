// Sequence sharding (context parallelism): the pieces that join scans of
// consecutive segments of one sequence into the scan of the whole sequence.
//
// The recurrence is linear in its state, so a segment run from a zero state
// and a zero left endpoint gives its local end state, and the true end state is
// that plus the segment's whole transition applied to what enters it
// ("When a Diagonal State Is Not Enough", sungsoo.github.io, Part 03: the state
// carried between chunks of the chunked form is the same composition):
//     K_in(k + 1) = Phi_k (K_in(k) + beta_0(k) W_in(k)) + hT_loc(k),
//     W_in(k + 1) = last write of segment k,
// Phi_k = prod over the segment of A_t (per mode: e^{a sum dt} and a rotation
// by the summed angle), beta_0(k) the left-endpoint weight of its first token.
// The backward is the mirror image: the adjoint entering the end of segment k
// is the full adjoint of the next segment's initial state,
//     dK_end(k) = dh0_loc(k + 1) + Phi_{k+1}^T dK_end(k + 1),
// and the last write of segment k receives beta_0(k + 1) times it.
//
// Kernels: the segment transition, the two combines (an ordered scan over the
// gathered per-segment values, elementwise over (b, h, mode, channel)), the
// adjoint of the boundary write (added to dx / dB of the segment's last token),
// and the fill of the trailing rows through which a segment's backward receives
// its end adjoint (one-hot C rows read the state out; their dy carries it).
#include "common.cuh"

namespace ssm {

namespace cpk {
constexpr int THREADS = 256;
}

// phi of mode m of head h from the segment's dt sum S (with per-token angles, ang_tok
// is the pair's summed angle): e^{a S} on a dynamic real row, e^{a L} on a static one,
// and e^{a S} times the rotation by the summed angle on a pair
__device__ __forceinline__ void cp_mode_phi(const Params &p, int h, int m, float S, float ang_tok,
                                            float &re, float &im) {
    const float a = -expf(p.A_log[h * p.ndec + (p.per_coord ? m : 0)]);
    im = 0.f;
    if (m < p.nr) {
        re = expf(a * (m < p.nst ? (float)p.L : S));   // static rows: e^{a} per token
    } else {
        const float ang = p.angle_tok ? ang_tok : p.theta[h * p.np + (m - p.nr)] * S;
        float sn, cs;
        sincosf(ang, &sn, &cs);
        const float mag = expf(a * S);
        re = mag * cs;
        im = mag * sn;
    }
}

__device__ __forceinline__ float cp_beta0(const Params &p, int b, int h) {
    if (!p.two_ep || p.L < 1) return 0.f;
    return (1.f - ld_io(p.lam, ix_lam(p, b, 0, h), p.bf16)) * ld_io(p.dt, ix_dt(p, b, 0, h), p.bf16);
}

// Phi of every (b, h, mode) of the segment ([B][H][nmode][2], (re, im)) and
// beta_0 ([B][H]).  One CTA per (b, h): the sums of dt (and of the per-token
// angles) over the segment in a fixed order, then one thread per mode.
__global__ void __launch_bounds__(cpk::THREADS) k_cp_transition(Params p, float *phi, float *beta0) {
    __shared__ float red[cpk::THREADS];
    __shared__ float th[64 * 8];   // per-token angle partial sums [pair][warp]
    const int bh = blockIdx.x, b = bh / p.H, h = bh - b * p.H;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    float s = 0.f;
    for (int t = tid; t < p.L; t += cpk::THREADS) s += ld_io(p.dt, ix_dt(p, b, t, h), p.bf16);
    red[tid] = s;
    // per-token angles: warp w sums tokens w, w + 8, ...; lane j (and j + 32) one pair
    if (p.angle_tok && p.np) {
        for (int j = lane; j < p.np; j += 32) {
            float a = 0.f;
            for (int t = warp; t < p.L; t += cpk::THREADS / 32) a += p.theta[ix_th(p, b, t, h, j)];
            th[j * 8 + warp] = a;
        }
    }
    __syncthreads();
    for (int w = cpk::THREADS / 2; w >= 1; w >>= 1) {
        if (tid < w) red[tid] += red[tid + w];
        __syncthreads();
    }
    const float S = red[0];
    const int nmode = p.nr + p.np;
    for (int m = tid; m < nmode; m += cpk::THREADS) {
        float ang = 0.f;
        if (p.angle_tok && m >= p.nr)
            for (int w = 0; w < cpk::THREADS / 32; ++w) ang += th[(m - p.nr) * 8 + w];
        float re, im;
        cp_mode_phi(p, h, m, S, ang, re, im);
        float *o = phi + ((long long)bh * nmode + m) * 2;
        o[0] = re;
        o[1] = im;
    }
    if (tid == 0) beta0[bh] = cp_beta0(p, b, h);
}

// The same for many heads (no per-token angles): one CTA per (32-head tile, b),
// the lane a head (so a warp's dt loads are contiguous), the warps interleaved
// tokens, their partial sums added in warp order.
__global__ void __launch_bounds__(cpk::THREADS) k_cp_transition_cols(Params p, float *phi,
                                                                     float *beta0) {
    constexpr int NW = cpk::THREADS / 32;
    __shared__ float part[NW][32];
    __shared__ float s_sum[32];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int h0 = blockIdx.x * 32, b = blockIdx.y, h = h0 + lane;
    float s = 0.f;
    if (h < p.H) {
#pragma unroll 4
        for (int t = warp; t < p.L; t += NW) s += ld_io(p.dt, ix_dt(p, b, t, h), p.bf16);
    }
    part[warp][lane] = s;
    __syncthreads();
    if (warp == 0) {
        float S = 0.f;
        for (int w = 0; w < NW; ++w) S += part[w][lane];
        s_sum[lane] = S;
        if (h < p.H) beta0[(long long)b * p.H + h] = cp_beta0(p, b, h);
    }
    __syncthreads();
    const int nmode = p.nr + p.np;
    const int nh = min(32, p.H - h0);
    for (int i = threadIdx.x; i < nh * nmode; i += blockDim.x) {
        const int hl = i / nmode, m = i - hl * nmode;
        float re, im;
        cp_mode_phi(p, h0 + hl, m, s_sum[hl], 0.f, re, im);
        float *o = phi + (((long long)b * p.H + h0 + hl) * nmode + m) * 2;
        o[0] = re;
        o[1] = im;
    }
}

// Unit (b, h, mode m, channel q): a real mode is one state row, a pair mode its
// (re, im) rows.
struct CpUnit {
    int b, h, m, q, n0;
    bool pair;
};
__device__ __forceinline__ CpUnit cp_unit(const Params &p, long long u) {
    const int nmode = p.nr + p.np;
    CpUnit c;
    c.q = (int)(u % p.P);
    long long r = u / p.P;
    c.m = (int)(r % nmode);
    r /= nmode;
    c.h = (int)(r % p.H);
    c.b = (int)(r / p.H);
    c.pair = c.m >= p.nr;
    c.n0 = c.pair ? p.nr + 2 * (c.m - p.nr) : c.m;
    return c;
}

// State and left endpoint entering segment `seg` from the gathered local end
// states hT_all / last writes wT_all ([nseg][B][H][N][P]), transitions phi_all
// ([nseg][B][H][nmode][2]) and beta0_all ([nseg][B][H]) of the segments before
// it, starting from h0 / w0 (NULL = zero).
__global__ void __launch_bounds__(cpk::THREADS)
    k_cp_state_combine(Params p, int seg, const float *hT_all, const float *wT_all,
                       const float *phi_all, const float *beta0_all, const float *h0,
                       const float *w0, float *h_in, float *w_in) {
    const int nmode = p.nr + p.np;
    const long long units = (long long)p.Bsz * p.H * nmode * p.P;
    const long long st = (long long)p.Bsz * p.H * p.N * p.P;   // one segment's state
    const long long bhs = (long long)p.Bsz * p.H;
    for (long long u = blockIdx.x * (long long)blockDim.x + threadIdx.x; u < units;
         u += (long long)gridDim.x * blockDim.x) {
        const CpUnit c = cp_unit(p, u);
        const long long i0 = ix_st(p, c.b, c.h, c.n0, c.q);
        const long long i1 = c.pair ? ix_st(p, c.b, c.h, c.n0 + 1, c.q) : i0;
        float hr = h0 ? h0[i0] : 0.f, hi = (c.pair && h0) ? h0[i1] : 0.f;
        float wr = w0 ? w0[i0] : 0.f, wi = (c.pair && w0) ? w0[i1] : 0.f;
        const long long bh = (long long)c.b * p.H + c.h;
        for (int k = 0; k < seg; ++k) {
            const float be = beta0_all[k * bhs + bh];
            const float *ph = phi_all + ((k * bhs + bh) * nmode + c.m) * 2;
            const float zr = fmaf(be, wr, hr), zi = fmaf(be, wi, hi);
            hr = fmaf(ph[0], zr, -ph[1] * zi) + hT_all[k * st + i0];
            hi = c.pair ? fmaf(ph[1], zr, ph[0] * zi) + hT_all[k * st + i1] : 0.f;
            wr = wT_all[k * st + i0];
            wi = c.pair ? wT_all[k * st + i1] : 0.f;
        }
        h_in[i0] = hr;
        w_in[i0] = wr;
        if (c.pair) {
            h_in[i1] = hi;
            w_in[i1] = wi;
        }
    }
}

// Adjoint entering the end of segment `seg` (and the adjoint of its last write)
// from the gathered local initial-state adjoints dh0_all ([nseg][B][H][N][P]) and
// transitions of the segments after it, starting from dhT (NULL = zero) at the
// end of the last segment.
__global__ void __launch_bounds__(cpk::THREADS)
    k_cp_adjoint_combine(Params p, int nseg, int seg, const float *dh0_all,
                         const float *phi_all, const float *beta0_all, const float *dhT,
                         float *dh_end, float *dw_end) {
    const int nmode = p.nr + p.np;
    const long long units = (long long)p.Bsz * p.H * nmode * p.P;
    const long long st = (long long)p.Bsz * p.H * p.N * p.P;
    const long long bhs = (long long)p.Bsz * p.H;
    for (long long u = blockIdx.x * (long long)blockDim.x + threadIdx.x; u < units;
         u += (long long)gridDim.x * blockDim.x) {
        const CpUnit c = cp_unit(p, u);
        const long long i0 = ix_st(p, c.b, c.h, c.n0, c.q);
        const long long i1 = c.pair ? ix_st(p, c.b, c.h, c.n0 + 1, c.q) : i0;
        float gr = dhT ? dhT[i0] : 0.f, gi = (c.pair && dhT) ? dhT[i1] : 0.f;
        const long long bh = (long long)c.b * p.H + c.h;
        for (int k = nseg - 1; k > seg; --k) {
            // full adjoint of segment k's initial state: its own part + Phi_k^T g
            const float *ph = phi_all + ((k * bhs + bh) * nmode + c.m) * 2;
            const float nr_ = fmaf(ph[0], gr, ph[1] * gi) + dh0_all[k * st + i0];
            const float ni_ = c.pair ? fmaf(-ph[1], gr, ph[0] * gi) + dh0_all[k * st + i1] : 0.f;
            gr = nr_;
            gi = ni_;
        }
        const float be = seg + 1 < nseg ? beta0_all[(seg + 1) * bhs + bh] : 0.f;
        dh_end[i0] = gr;
        dw_end[i0] = be * gr;
        if (c.pair) {
            dh_end[i1] = gi;
            dw_end[i1] = be * gi;
        }
    }
}

// dW of the segment's last token (t = L - 1) receives dw_end: dx += B^T dw_end per
// head, dB += sum over the group's heads of dw_end u^T.  Thread (b, h, r, q) for dx,
// then (b, g, r, n) for dB.
__global__ void __launch_bounds__(cpk::THREADS) k_cp_write_adjoint(Params p, const float *dw_end) {
    // dx of the last token: one thread per (b, h, r, q), the sum over the state rows
    const int t = p.L - 1;
    const long long nx = (long long)p.Bsz * p.H * p.R * p.P;
    for (long long u = blockIdx.x * (long long)blockDim.x + threadIdx.x; u < nx;
         u += (long long)gridDim.x * blockDim.x) {
        const int q = (int)(u % p.P);
        long long r_ = u / p.P;
        const int r = (int)(r_ % p.R);
        r_ /= p.R;
        const int h = (int)(r_ % p.H), b = (int)(r_ / p.H), g = h / p.hpg;
        float acc = 0.f;
        for (int n = 0; n < p.N; ++n)
            acc = fmaf(ld_io(p.Bm, ix_B(p, b, t, g, r, n), p.bf16), dw_end[ix_st(p, b, h, n, q)], acc);
        const long long ix = ix_x(p, b, t, h, r, q);
        st_io(p.dx, ix, ld_io(p.dx, ix, p.bf16) + acc, p.bf16);
    }
}

// dB of the last token: one block per (b, g, r, n), the sum over the group's
// (head, channel) pairs in a fixed order (thread-strided partials, a shuffle
// tree per warp, then the warps in order)
__global__ void __launch_bounds__(cpk::THREADS) k_cp_write_adjoint_b(Params p, const float *dw_end) {
    __shared__ float part[cpk::THREADS / 32];
    const int t = p.L - 1;
    int u = blockIdx.x;
    const int n = u % p.N;
    u /= p.N;
    const int r = u % p.R;
    u /= p.R;
    const int g = u % p.G, b = u / p.G;
    const int cnt = p.hpg * p.P;
    float acc = 0.f;
    for (int i = threadIdx.x; i < cnt; i += blockDim.x) {
        const int h = g * p.hpg + i / p.P, q = i % p.P;
        acc = fmaf(dw_end[ix_st(p, b, h, n, q)], ld_io(p.x, ix_x(p, b, t, h, r, q), p.bf16), acc);
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = acc;
    __syncthreads();
    if (threadIdx.x == 0) {
        float sum = 0.f;
        for (int w = 0; w < cpk::THREADS / 32; ++w) sum += part[w];
        const long long ib = ix_B(p, b, t, g, r, n);
        st_io(p.dBm, ib, ld_io(p.dBm, ib, p.bf16) + sum, p.bf16);
    }
}

// Trailing rows t = L .. L + nv - 1 of a segment's buffers (p.L = the segment's
// own length, the buffers hold L + nv tokens): zero dt, x, B, lambda 1 (static
// angles, no static rows), so the state passes through unchanged and nothing is
// written; C row o = 0 of trailing token L + s N + k is e_k (the others zero),
// and its dy carries part s of dh_end[:, k, :] (bf16: s = 0 the bf16 value,
// s = 1 the remainder; fp32: one part).  The backward over L + nv tokens then
// receives dh_end as the adjoint of the segment's end state; every gradient a
// trailing row adds to the parameters is weighted by its dt (zero) or its input
// (zero).
__global__ void __launch_bounds__(cpk::THREADS) k_cp_fill_tail(Params p, int nv, const float *dh_end) {
    // one block per trailing row (b, v); its threads take each field's elements with
    // the innermost index fastest, so the stores of a warp are contiguous
    const int nsets = nv / p.N;
    const int rows = p.Bsz * nv;
    const int nx = p.H * p.R * p.P, ny = p.H * p.O * p.P;
    const int nb = p.G * p.R * p.N, nc = p.G * p.O * p.N;
    const bool all = p.x != nullptr;   // else only the dy rows
    for (int row = blockIdx.x; row < rows; row += gridDim.x) {
        const int b = row / nv, v = row - b * nv, t = p.L + v;
        const int s = v / p.N, k = v - s * p.N;
        // dt = 0 and lambda = 1
        for (int h = threadIdx.x; all && h < p.H; h += blockDim.x) {
            st_io((void *)p.dt, ix_dt(p, b, t, h), 0.f, p.bf16);
            if (p.two_ep) st_io((void *)p.lam, ix_lam(p, b, t, h), 1.f, p.bf16);
        }
        // x = 0
        for (int i = threadIdx.x; all && i < nx; i += blockDim.x) {
            const int q = i % p.P, r1 = i / p.P, rr = r1 % p.R, h = r1 / p.R;
            st_io((void *)p.x, ix_x(p, b, t, h, rr, q), 0.f, p.bf16);
        }
        // dy: in target rank 0 of trailing row v = s N + k, row k of the end adjoint
        // (s = 0: its io-precision value; s = 1: the remainder), zero elsewhere
        for (int i = threadIdx.x; i < ny; i += blockDim.x) {
            const int q = i % p.P, r1 = i / p.P, o = r1 % p.O, h = r1 / p.O;
            float val = 0.f;
            if (o == 0) {
                const float d = dh_end ? dh_end[ix_st(p, b, h, k, q)] : 0.f;
                const float hi = p.bf16 ? __bfloat162float(__float2bfloat16_rn(d)) : d;
                val = (nsets == 1 || s == 0) ? hi : d - hi;
            }
            st_io((void *)p.dy, ix_y(p, b, t, h, o, q), val, p.bf16);
        }
        // B = 0; C = e_k in target rank 0
        for (int i = threadIdx.x; all && i < nb; i += blockDim.x) {
            const int n = i % p.N, r1 = i / p.N, rr = r1 % p.R, g = r1 / p.R;
            st_io((void *)p.Bm, ix_B(p, b, t, g, rr, n), 0.f, p.bf16);
        }
        for (int i = threadIdx.x; all && i < nc; i += blockDim.x) {
            const int n = i % p.N, r1 = i / p.N, o = r1 % p.O, g = r1 / p.O;
            st_io((void *)p.Cm, ix_C(p, b, t, g, o, n), (o == 0 && n == k) ? 1.f : 0.f, p.bf16);
        }
    }
}

static int cp_blocks(long long units) {
    long long b = (units + cpk::THREADS - 1) / cpk::THREADS;
    if (b > 148 * 16) b = 148 * 16;
    return b < 1 ? 1 : (int)b;
}

cudaError_t cp_transition(const Params &p, float *phi, float *beta0, cudaStream_t st) {
    if (p.Bsz * p.H == 0) return cudaSuccess;
    if (p.H >= 256 && !(p.angle_tok && p.np)) {   // many heads: a CTA per 32-head tile
        k_cp_transition_cols<<<dim3((p.H + 31) / 32, p.Bsz), cpk::THREADS, 0, st>>>(p, phi, beta0);
        profile_mark(st, "k_cp_transition_cols");
    } else {
        k_cp_transition<<<p.Bsz * p.H, cpk::THREADS, 0, st>>>(p, phi, beta0);
        profile_mark(st, "k_cp_transition");
    }
    return cudaGetLastError();
}

cudaError_t cp_state_combine(const Params &p, int seg, const float *hT_all, const float *wT_all,
                             const float *phi_all, const float *beta0_all, const float *h0,
                             const float *w0, float *h_in, float *w_in, cudaStream_t st) {
    const long long units = (long long)p.Bsz * p.H * (p.nr + p.np) * p.P;
    k_cp_state_combine<<<cp_blocks(units), cpk::THREADS, 0, st>>>(p, seg, hT_all, wT_all, phi_all,
                                                                  beta0_all, h0, w0, h_in, w_in);
    profile_mark(st, "k_cp_state_combine");
    return cudaGetLastError();
}

cudaError_t cp_adjoint_combine(const Params &p, int nseg, int seg, const float *dh0_all,
                               const float *phi_all, const float *beta0_all, const float *dhT,
                               float *dh_end, float *dw_end, cudaStream_t st) {
    const long long units = (long long)p.Bsz * p.H * (p.nr + p.np) * p.P;
    k_cp_adjoint_combine<<<cp_blocks(units), cpk::THREADS, 0, st>>>(p, nseg, seg, dh0_all, phi_all,
                                                                    beta0_all, dhT, dh_end, dw_end);
    profile_mark(st, "k_cp_adjoint_combine");
    return cudaGetLastError();
}

cudaError_t cp_write_adjoint(const Params &p, const float *dw_end, cudaStream_t st) {
    if (p.L < 1) return cudaSuccess;
    const long long units = (long long)p.Bsz * p.H * p.R * p.P;
    k_cp_write_adjoint<<<cp_blocks(units), cpk::THREADS, 0, st>>>(p, dw_end);
    profile_mark(st, "k_cp_write_adjoint");
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const long long nbo = (long long)p.Bsz * p.G * p.R * p.N;
    if (nbo == 0) return cudaSuccess;
    k_cp_write_adjoint_b<<<(unsigned)nbo, cpk::THREADS, 0, st>>>(p, dw_end);
    profile_mark(st, "k_cp_write_adjoint_b");
    return cudaGetLastError();
}

cudaError_t cp_fill_tail(const Params &p, int nv, const float *dh_end, cudaStream_t st) {
    const long long rows = (long long)nv * p.Bsz;
    if (rows == 0) return cudaSuccess;
    k_cp_fill_tail<<<(int)(rows < 148 * 16 ? rows : 148 * 16), cpk::THREADS, 0, st>>>(p, nv, dh_end);
    profile_mark(st, "k_cp_fill_tail");
    return cudaGetLastError();
}

}  // namespace ssm
