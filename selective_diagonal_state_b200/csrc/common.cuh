// Shared definitions of the sm_100a selective-diagonal-scan kernels.
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace ssm {

// Thread/row geometry of the SIMT scan kernels (chosen on the host).
//  PP: padded head dim (power of two, lanes over p)   NQ: row-groups per head
//  HC: heads per CTA    T: tokens staged in shared memory per block
struct Geometry {
    int PP, NQ, HC, T;
};

struct Params {
    // sizes
    int Bsz, L, H, P, G, nr, np, N, R, O, ndec, hpg;
    int two_ep, per_coord, bf16;
    int angle_tok;  // rotation angles given per token: theta / dtheta are [B][L][H][np]
    int nst;        // the first nst real rows are static (transition e^{a} whatever dt)
    int zoh;        // exact zero-order-hold write (two_endpoint == 0, nst == 0)
    // element strides (batch, time, head-or-group)
    long long sx[3], sy[3], sB[3], sC[3], sdt[3], slam[3];
    // inputs
    const void *x, *dt, *Bm, *Cm, *lam, *dy;
    const float *A_log, *theta, *D, *h0, *w0;
    // forward outputs
    void *y;
    float *hT, *wT;
    // output gate of the mixer (null: none): y_g = y * silu(z), z in y's layout; the
    // pre-gate y is kept in ypre when set
    const void *gz;
    void *ypre;
    // backward outputs
    void *dx, *ddt, *dBm, *dCm, *dlam;
    float *dA_log, *dtheta, *dD, *dh0, *dw0;
    // backward workspace (fp32)
    float *ws_dC;   // [B][L][H][O][N]   per-head dC_t = dy_t H_t^T
    float *ws_gbu;  // [B][L][H][R][N]   sum_p Gbar_t[n,p] u_t[r,p]
    float *ws_tok;  // [B][L][H][2]      (dsigma_t, <dy_t, C_t W_t>)
    float *ws_M2;   // [B][L][H][O][R]   <dy_t[o,:], u_t[r,:]>
    float *ws_par;  // [B][H][NPAR]      per-unit partials of dA, dtheta, dD, dbeta_0
    float *ws_ddt;  // [B][L][H]         local decay part of ddt (within a time block)
    float *ws_blk;  // [B][H][NTB][4 nmode + 2]  per time block: totals and local sums
    float *ws_blkc; // [B][H][NTB]       ddt offset of each time block (carried part)
    // chunk states and exact decay-gradient carries at 64-token chunk boundaries
    // (tensor-core chain; the forward uses ws_kp and ws_ce):
    float *ws_kp;   // [B][H][NC] 32 KB: pre-state K entering every chunk (K_{-1} = h0 + beta_0 w0)
    float *ws_qb;   // [B][H][NC][4][N]  per-row sum_p conj(Gbar) A K_prev at chunk starts (4 partials over p)
    float *ws_gc;   // [B][H][NC] 32 KB: the adjoint carried into each chunk (hi / lo tiles)
    float *ws_ce;   // [B][H][NC][128][2] full-chunk decay e^{lam S_63} per mode (re, im)
    // forward chain: fp32 state carried from chunk c to c + 1 through two slots per
    // (b, h), and the count of chunks of (b, h) whose outgoing state is in place
    float *ws_ring; // [2][B][H][4][4][128][4] carry slots (row-contiguous per 4 columns)
    int *ws_flag;   // [B][H] counters, then [0] the next work item (ticket) and [1] the
                    // abort word of this call (the backward carries its adjoint the same way)
    long long wait_limit;   // polls of a carry counter before a wait gives up
    int nc;         // number of 64-token chunks
    // device-side choice between two launched kernel chains: a kernel runs
    // only when (*gate != 0) == gate_on (no gate: always)
    const int *gate;
    int gate_on;
    // the backward takes ws_kp / ws_ce as written by the forward (not recomputed)
    int states_ready;
    // per-chunk products a training forward saves for the backward (null: not saved):
    unsigned char *sv_P;    // [B][H][NC] 8 KB: masked scores P^T as bf16 operand tiles
    unsigned char *sv_Bh;   // [B][H][NC] 16 KB: chunk-end folded B (bf16 operand tile)
    float *sv_corr;         // [B][H][NC][64] D - beta_{t+1} C_t . B_t
    // scalar-decay chain backward (chunks of 128 / R tokens):
    float *sd_tok;          // [B][L][H][3] dsigma_t, diag_t (the gamma_t part), drho_t
    float *sd_par;          // [B][H][NC][2] per chunk: sum_t dt_t drho_t, sum <dy, x>
    float *sd_db0;          // [B][H] dbeta_0 = <dL/dK_{-1}, w0>
    float *sd_dBh, *sd_dCh; // [B][L][H][R or O][N] fp32 per-head dB / dC (several heads per group)
    // scalar-decay forward, segments of sd_G chunks: per (segment, b, h) the state the
    // segment adds, then the state entering it ([nseg][B][H] 32 KB, in place), the
    // segment's decay [nseg][B][H], and one 32 KB carry slot per CTA
    float *sd_seg, *sd_sege, *sd_priv;
    int sd_G, sd_nseg;
    Geometry geo;
};

__device__ __forceinline__ bool gated_off(const Params &p) {
    return p.gate && ((*p.gate != 0) != (p.gate_on != 0));
}

// per-unit partial slots in ws_par
__host__ __device__ inline int npar_of(const Params &p) { return p.ndec + p.np + 2; }

__device__ __forceinline__ float ld_io(const void *ptr, long long i, int bf16) {
    if (bf16) return __bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(ptr)[i]);
    return reinterpret_cast<const float *>(ptr)[i];
}
__device__ __forceinline__ void st_io(void *ptr, long long i, float v, int bf16) {
    if (bf16)
        reinterpret_cast<__nv_bfloat16 *>(ptr)[i] = __float2bfloat16_rn(v);
    else
        reinterpret_cast<float *>(ptr)[i] = v;
}

__device__ __forceinline__ long long ix_x(const Params &p, int b, int t, int h, int r, int q) {
    return b * p.sx[0] + t * p.sx[1] + h * p.sx[2] + (long long)r * p.P + q;
}
__device__ __forceinline__ long long ix_y(const Params &p, int b, int t, int h, int o, int q) {
    return b * p.sy[0] + t * p.sy[1] + h * p.sy[2] + (long long)o * p.P + q;
}
__device__ __forceinline__ long long ix_B(const Params &p, int b, int t, int g, int r, int n) {
    return b * p.sB[0] + t * p.sB[1] + g * p.sB[2] + (long long)r * p.N + n;
}
__device__ __forceinline__ long long ix_C(const Params &p, int b, int t, int g, int o, int n) {
    return b * p.sC[0] + t * p.sC[1] + g * p.sC[2] + (long long)o * p.N + n;
}
__device__ __forceinline__ long long ix_dt(const Params &p, int b, int t, int h) {
    return b * p.sdt[0] + t * p.sdt[1] + h * p.sdt[2];
}
__device__ __forceinline__ long long ix_lam(const Params &p, int b, int t, int h) {
    return b * p.slam[0] + t * p.slam[1] + h * p.slam[2];
}
// per-token rotation angle of pair j (dense [B][L][H][np])
__device__ __forceinline__ long long ix_th(const Params &p, int b, int t, int h, int j) {
    return (((long long)b * p.L + t) * p.H + h) * p.np + j;
}
__device__ __forceinline__ long long ix_st(const Params &p, int b, int h, int n, int q) {
    return (((long long)b * p.H + h) * p.N + n) * p.P + q;
}
// dense per-head workspace [B][L][H][K][N]
__device__ __forceinline__ long long ix_wsk(const Params &p, int b, int t, int h, int k, int K,
                                            int n) {
    return ((((long long)b * p.L + t) * p.H + h) * K + k) * p.N + n;
}
__device__ __forceinline__ long long ix_bth(const Params &p, int b, int t, int h) {
    return ((long long)b * p.L + t) * p.H + h;
}

// decay slot of state row n: per-head mode has one slot; per-coordinate mode
// has one per real row followed by one per rotation pair
__device__ __forceinline__ int dec_slot(const Params &p, int n) {
    if (!p.per_coord) return 0;
    return n < p.nr ? n : p.nr + (n - p.nr) / 2;
}

// Slot layout: thread-row-group q owns NS = NR + 2*NPR consecutive slots:
// real rows q, q+NQ, ... (NR of them) then pairs q, q+NQ, ... as (re, im).
// slot_of maps a state row to its slot index in [0, NQ*NS).
template <int NR, int NPR>
__device__ __forceinline__ int slot_of(int n, int nr, int NQ) {
    constexpr int NS = NR + 2 * NPR;
    if (n < nr) return (n % NQ) * NS + n / NQ;
    int j = (n - nr) >> 1, c = (n - nr) & 1;
    return (j % NQ) * NS + NR + 2 * (j / NQ) + c;
}
// inverse: state row of slot s within group q (or -1 for a padding slot)
template <int NR, int NPR>
__device__ __forceinline__ int row_of(int q, int s, int nr, int np, int NQ) {
    if (s < NR) {
        int n = q + s * NQ;
        return n < nr ? n : -1;
    }
    int j = q + ((s - NR) >> 1) * NQ, c = (s - NR) & 1;
    return j < np ? nr + 2 * j + c : -1;
}

// Sum each of K register values over the S lanes that share everything but p
// (S = 1, 16 or 32 consecutive lanes).  Afterwards, for K >= S lane l holds
// the totals of values [l*K/S, (l+1)*K/S) in v[0..K/S); for K < S lane l holds
// the total of value l/(S/K) in v[0].
template <int K, int S>
__device__ __forceinline__ void xreduce(float (&v)[K], int lane) {
    if constexpr (S > 1) {
        constexpr unsigned FULL = 0xffffffffu;
        int cur = K;
#pragma unroll
        for (int m = S / 2; m >= 1; m >>= 1) {
            if (cur > 1) {
                const bool up = (lane & m) != 0;
                const int hlf = cur / 2;
#pragma unroll
                for (int i = 0; i < K / 2; ++i) {
                    if (i < hlf) {
                        float send = up ? v[i] : v[i + hlf];
                        float keep = up ? v[i + hlf] : v[i];
                        v[i] = keep + __shfl_xor_sync(FULL, send, m);
                    }
                }
                cur = hlf;
            } else {
                v[0] += __shfl_xor_sync(FULL, v[0], m);
            }
        }
    }
}

// ---- exact zero-order hold --------------------------------------------------
// phi1(mu) = (e^mu - 1) / mu and phi1'(mu) = (e^mu (mu - 1) + 1) / mu^2 of a
// complex mu = (mr, mi), by their Taylor series for |mu| < 1/2 (where the
// closed forms cancel) and the closed forms above it.
__device__ __forceinline__ void cmulf(float ar, float ai, float br, float bi, float &cr, float &ci) {
    cr = ar * br - ai * bi;
    ci = ar * bi + ai * br;
}
__device__ __forceinline__ void zoh_phi(float mr, float mi, float &f1r, float &f1i, float &fdr,
                                        float &fdi) {
    if (mr * mr + mi * mi < 0.25f) {
        // sum_k mu^k / (k + 1)!  and  sum_k (k + 1) mu^k / (k + 2)!, 12 terms
        float pr = 1.f, pi = 0.f;   // mu^k
        f1r = f1i = fdr = fdi = 0.f;
        float inv1 = 1.f, inv2 = 0.5f;   // 1 / (k + 1)!, 1 / (k + 2)!
#pragma unroll
        for (int k = 0; k < 12; ++k) {
            f1r = fmaf(inv1, pr, f1r);
            f1i = fmaf(inv1, pi, f1i);
            fdr = fmaf((k + 1) * inv2, pr, fdr);
            fdi = fmaf((k + 1) * inv2, pi, fdi);
            float nr, ni;
            cmulf(pr, pi, mr, mi, nr, ni);
            pr = nr;
            pi = ni;
            inv1 *= 1.f / (float)(k + 2);
            inv2 *= 1.f / (float)(k + 3);
        }
        return;
    }
    float sn, cs;
    sincosf(mi, &sn, &cs);
    const float ex = expf(mr);
    const float s2 = sinf(0.5f * mi);
    // e^mu - 1 without cancellation in its real part
    const float er = fmaf(expm1f(mr), cs, -2.f * s2 * s2), ei = ex * sn;
    const float d = 1.f / (mr * mr + mi * mi);   // 1 / |mu|^2
    // (e^mu - 1) conj(mu) / |mu|^2
    f1r = (er * mr + ei * mi) * d;
    f1i = (ei * mr - er * mi) * d;
    // phi1'(mu) = (e^mu - phi1(mu)) / mu
    const float nr = ex * cs - f1r, ni = ex * sn - f1i;
    fdr = (nr * mr + ni * mi) * d;
    fdi = (ni * mr - nr * mi) * d;
}

// The same for a real argument: phi1(m) and phi1'(m).
__device__ __forceinline__ void zoh_phi_real(float m, float &f1, float &fd) {
    if (m * m < 0.25f) {
        float pw = 1.f, inv1 = 1.f, inv2 = 0.5f;
        f1 = fd = 0.f;
#pragma unroll
        for (int k = 0; k < 12; ++k) {
            f1 = fmaf(inv1, pw, f1);
            fd = fmaf((k + 1) * inv2, pw, fd);
            pw *= m;
            inv1 *= 1.f / (float)(k + 2);
            inv2 *= 1.f / (float)(k + 3);
        }
        return;
    }
    const float d = 1.f / m;
    f1 = expm1f(m) * d;
    fd = (expf(m) - f1) * d;
}

// Timing hook (defined in abi.cu): call right after every kernel launch with
// the kernel's name.
void profile_mark(cudaStream_t st, const char *name);

}  // namespace ssm
