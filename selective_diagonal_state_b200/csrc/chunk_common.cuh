// Pieces shared by the chunked tensor-core kernels (64-token chunks of four
// 16-token sub-blocks, bf16 operands, fp32 accumulation): sizes, the fp32
// scratch map, bf16 packing, reads of 128-byte-swizzled B/C tiles, mode
// constants slots, and the host-side TMA descriptor encoder.
#pragma once
#include <cuda.h>

#include <type_traits>

#include "common.cuh"
#include "umma.cuh"

namespace ssm {
namespace chunkc {

using namespace umma;

constexpr int Q = 64;
constexpr int NSB = 4;
constexpr int NP = 128;   // state rows (K) padded
constexpr int PD = 64;    // head dim
constexpr uint32_t WAIT_LIMIT = 1u << 22;

// fp32 scratch (float offsets from SM_F32)
constexpr int F_S = 0, F_SIG = 64, F_BN = 128, F_CORR = 192, F_DT = 256, F_LAM = 328;
constexpr int F_CP = 400;                 // [4][64] corr partials
constexpr int F_A2 = 656;                 // [128] decay * log2(e) per mode
constexpr int F_W = 784;                  // [128] rotation frequency per mode
constexpr int F_KRE = 912;                // [13][128] mode constants, real part
constexpr int F_KIM = F_KRE + 13 * 128;   // [13][128] imaginary part
constexpr int F_END = F_KIM + 13 * 128;
// per-token rotation angles (p.angle_tok): inclusive prefix over the chunk's tokens,
// pair-major with a padded row, Theta[j][t] at F_TH + j * TH_LD + t
constexpr int TH_LD = 65;
constexpr int F_TH = F_END;
constexpr int F_END_TH = F_TH + 64 * TH_LD;

constexpr uint32_t KM_LBO = 128, KM_SBO = 2048;  // K-major tiles with K = 128

__device__ __forceinline__ uint32_t bi_off(int i) {
    return i == 0 ? 0u : (i == 1 ? 4096u : (i == 2 ? 12288u : 24576u));
}
// mode-constant slots: F[i][j] = prod_{k=i}^{j-1} E_k (0 <= i < j <= 4), G[i] = conj(F[0][i])
__device__ __forceinline__ int fslot(int i, int j) {
    return (i == 0 ? 0 : (i == 1 ? 4 : (i == 2 ? 7 : 9))) + (j - i - 1);
}
__device__ __forceinline__ int gslot(int i) { return 10 + (i - 1); }

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}
__device__ __forceinline__ void st16(unsigned char *base, uint32_t off, const float (&v)[8]) {
    uint4 w;
    w.x = pack_bf16(v[0], v[1]);
    w.y = pack_bf16(v[2], v[3]);
    w.z = pack_bf16(v[4], v[5]);
    w.w = pack_bf16(v[6], v[7]);
    *reinterpret_cast<uint4 *>(base + off) = w;
}
// store v as bf16 hi (at hi + off) and the bf16 residual v - hi (at lo + off)
__device__ __forceinline__ void st16_split(unsigned char *hi, unsigned char *lo, uint32_t off,
                                           const float (&v)[8]) {
    float h[8], l[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        h[i] = __bfloat162float(__float2bfloat16_rn(v[i]));
        l[i] = v[i] - h[i];
    }
    st16(hi, off, h);
    st16(lo, off, l);
}
__device__ __forceinline__ float bf(const unsigned char *p) {
    return __bfloat162float(*reinterpret_cast<const __nv_bfloat16 *>(p));
}
// 8 consecutive state rows r0..r0+7 of token t from a raw B/C tile
// (two 64-row halves, each 64 tokens x 128 bytes with the 128-byte swizzle).
__device__ __forceinline__ void ld_rows8(const unsigned char *tile, int t, int r0, float (&v)[8]) {
    const uint4 w = *reinterpret_cast<const uint4 *>(tile + (r0 >> 6) * 8192 +
                                                     off_sw128(t, r0 & 63));
    const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        v[2 * i] = __uint_as_float(u[i] << 16);
        v[2 * i + 1] = __uint_as_float(u[i] & 0xffff0000u);
    }
}
__device__ __forceinline__ float ld_row1(const unsigned char *tile, int t, int r) {
    return bf(tile + (r >> 6) * 8192 + off_sw128(t, r & 63));
}

__device__ __forceinline__ void st_row1(unsigned char *tile, int t, int r, float v) {
    *reinterpret_cast<__nv_bfloat16 *>(tile + (r >> 6) * 8192 + off_sw128(t, r & 63)) =
        __float2bfloat16_rn(v);
}

// 2^x with the hardware approximation (operands are rounded to bf16 afterwards)
__device__ __forceinline__ float ex2_fast(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// complex multiply (a + ib)(c + id)
__device__ __forceinline__ void cmul(float a, float b, float c, float d, float &re, float &im) {
    re = fmaf(a, c, -b * d);
    im = fmaf(a, d, b * c);
}

// ---- per-chunk token quantities and mode constants ----------------------------
// One chunk's dt / lambda of tokens t0 .. t0+64, held in registers of threads
// 0..64 between the load and the use (so that a persistent kernel can fetch
// the next chunk's while it works on this one).
// dt / lambda of one token (bf16 bits), loaded one chunk ahead: the values
// are converted only when chunk_tokens_from stores them, so the loads stay in
// flight until then.
struct TokPrefetch {
    unsigned short dv, lv;
};
__device__ __forceinline__ TokPrefetch tok_load(const Params &p, int b, int h, int t0) {
    TokPrefetch r{0, 0x3f80};   // dt 0, lambda 1
    const int i = threadIdx.x, t = t0 + i;
    if (i < Q + 1 && t < p.L) {
        r.dv = __ldg(reinterpret_cast<const unsigned short *>(p.dt) + ix_dt(p, b, t, h));
        if (p.two_ep) r.lv = __ldg(reinterpret_cast<const unsigned short *>(p.lam) + ix_lam(p, b, t, h));
    }
    return r;
}
// Writes the inclusive prefix S_t (F_S) and, with `want_sigma`, sigma_t (F_SIG)
// and beta_{t+1} (F_BN) from prefetched dt / lambda.  Call with all threads of
// the block (>= 96); contains barriers.
__device__ __forceinline__ void chunk_tokens_from(const Params &p, float *f32, int t0,
                                                  const TokPrefetch &r, bool want_sigma) {
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid < Q + 1) {
        f32[F_DT + tid] = __uint_as_float((uint32_t)r.dv << 16);
        f32[F_LAM + tid] = __uint_as_float((uint32_t)r.lv << 16);
    }
    __syncthreads();
    if (warp == 0) {
        const float d0 = f32[F_DT + 2 * lane], d1 = f32[F_DT + 2 * lane + 1];
        float v = d0 + d1;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float u = __shfl_up_sync(0xffffffffu, v, o);
            if (lane >= o) v += u;
        }
        f32[F_S + 2 * lane] = v - d1;
        f32[F_S + 2 * lane + 1] = v;
    } else if (want_sigma && (warp == 1 || warp == 2)) {
        const int t = (warp - 1) * 32 + lane;
        const float dv = f32[F_DT + t], lv = f32[F_LAM + t];
        const float bn =
            (t0 + t + 1 < p.L) ? (1.f - f32[F_LAM + t + 1]) * f32[F_DT + t + 1] : 0.f;
        f32[F_SIG + t] = fmaf(lv, dv, bn);
        f32[F_BN + t] = bn;
    }
    __syncthreads();
}
// Loads dt / lambda of tokens t0 .. t0+64 and writes F_S (and F_SIG, F_BN).
__device__ __forceinline__ void chunk_tokens(const Params &p, float *f32, int b, int h, int t0,
                                             bool want_sigma) {
    const TokPrefetch r = tok_load(p, b, h, t0);
    chunk_tokens_from(p, f32, t0, r, want_sigma);
}

// sin / cos of x after reducing it to [-pi, pi] (the fast intrinsic is only
// accurate near zero).
__device__ __forceinline__ void sincos_red(float x, float *sn, float *cs) {
    const float r = fmaf(-6.28318530717958648f, rintf(x * 0.159154943091895336f), x);
    __sincosf(r, sn, cs);
}

// Per-token angles of the chunk starting at token t0 into F_TH: Theta[j][t] = sum of
// theta over tokens t0 .. t0 + t (tokens past L add nothing).  All threads; ends with
// a barrier.
__device__ __forceinline__ void chunk_angles(const Params &p, float *f32, int b, int h, int t0) {
    const int np = p.np;
    float *th = f32 + F_TH;
    for (int i = threadIdx.x; i < 64 * np; i += blockDim.x) {   // coalesced over the pairs
        const int t = i / np, j = i - t * np;
        th[j * TH_LD + t] = (t0 + t < p.L) ? __ldg(p.theta + ix_th(p, b, t0 + t, h, j)) : 0.f;
    }
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
    for (int j = warp; j < np; j += nw) {   // a warp per pair: lane l takes tokens 2l, 2l + 1
        float *row = th + j * TH_LD;
        const float a0 = row[2 * lane], a1 = row[2 * lane + 1];
        float v = a0 + a1;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float u = __shfl_up_sync(0xffffffffu, v, o);
            if (lane >= o) v += u;
        }
        const float base = v - (a0 + a1);
        row[2 * lane] = base + a0;
        row[2 * lane + 1] = base + a0 + a1;
    }
    __syncthreads();
}
// Theta of pair j at chunk token t (t = -1: the chunk start)
__device__ __forceinline__ float th_at(const float *f32, int j, int t) {
    return t < 0 ? 0.f : f32[F_TH + j * TH_LD + t];
}
// Rotation angle of pair j from chunk token tr to token t (tr = -1: the chunk start):
// the pair's frequency times the step sum ds between them, or (TOK, per-token angles)
// the angles summed over (tr, t].  The kernels are instantiated once per angle mode.
template <bool TOK>
__device__ __forceinline__ float pair_angle(const float *f32, int j, float w, float ds, int t,
                                           int tr) {
    if constexpr (TOK)
        return th_at(f32, j, t) - th_at(f32, j, tr);
    else
        return w * ds;
}
template <bool TOK>
__device__ __forceinline__ void pair_sincos(float ang, float *sn, float *cs) {
    if constexpr (TOK)
        sincos_red(ang, sn, cs);   // per-token angles can be any size
    else
        __sincosf(ang, sn, cs);
}

// Exact zero-order-hold write (ZOH): the write of chunk token t on mode m is
// scaled by Z = dt phi1(dt a + i phi), phi1(z) = (e^z - 1) / z, in place of sigma_t
// (the Euler form's dt), phi the token's rotation angle on a pair (dt theta_j, or
// the token's own angle with per-token angles) and 0 on a real row.  Tokens past
// the sequence end have dt = 0 and so Z = 0.
__device__ __forceinline__ float zoh_real(const float *f32, int m, int t) {
    const float dv = f32[F_DT + t];
    float f1, fd;
    zoh_phi_real(dv * f32[F_A2 + m] * 0.6931471805599453f, f1, fd);
    return dv * f1;
}
// the token's own rotation angle on pair j (m its mode, w its frequency)
template <bool TOK>
__device__ __forceinline__ float tok_angle(const float *f32, int j, float w, int t) {
    if constexpr (TOK)
        return th_at(f32, j, t) - th_at(f32, j, t - 1);
    else
        return f32[F_DT + t] * w;
}
// (b0 + i b1) <- Z (b0 + i b1) on pair j of mode m
template <bool TOK>
__device__ __forceinline__ void zoh_pair(const float *f32, int m, int j, int t, float &b0,
                                         float &b1) {
    const float dv = f32[F_DT + t];
    float f1r, f1i, fdr, fdi;
    zoh_phi(dv * f32[F_A2 + m] * 0.6931471805599453f, tok_angle<TOK>(f32, j, f32[F_W + m], t), f1r,
            f1i, fdr, fdi);
    const float zr = dv * f1r, zi = dv * f1i;
    const float r = fmaf(zr, b0, -zi * b1);
    b1 = fmaf(zi, b0, zr * b1);
    b0 = r;
}

// Per-mode decay over each sub-block, E_k = e^{lam dS_k}, the products
// F[i][j] = prod_{k=i}^{j-1} E_k (E_k itself is F[k][k+1]) and
// G_i = conj(F[0][i]) into the F_KRE / F_KIM slots.  Four consecutive lanes
// take one mode, lane k its sub-block k; the four factors are exchanged by
// shuffles inside the group.  Needs F_S, F_A2, F_W; ends with a barrier.
template <bool TOK>
__device__ __forceinline__ void chunk_mode_constants(const Params &p, float *f32) {
    const int nmode = p.nr + p.np;
    for (int it = threadIdx.x; it < 4 * nmode; it += blockDim.x) {
        const int m = it >> 2, k = it & 3;
        const unsigned gm = 0xfu << (threadIdx.x & 28);   // the four lanes of this mode
        const float a2 = f32[F_A2 + m], w = f32[F_W + m];
        const float lo = k == 0 ? 0.f : f32[F_S + 16 * k - 1];
        const float ds = f32[F_S + 16 * k + 15] - lo;
        const float mag = ex2_fast(a2 * ds);
        float er = mag, ei = 0.f;
        if (m >= p.nr) {
            float sn, cs;
            sincos_red(pair_angle<TOK>(f32, m - p.nr, w, ds, 16 * k + 15, 16 * k - 1), &sn, &cs);
            er = mag * cs;
            ei = mag * sn;
        }
        float Er[4], Ei[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            Er[q] = __shfl_sync(gm, er, q, 4);
            Ei[q] = __shfl_sync(gm, ei, q, 4);
        }
        float *fr = f32 + F_KRE + m, *fi = f32 + F_KIM + m;
        fr[fslot(k, k + 1) * NP] = er;
        fi[fslot(k, k + 1) * NP] = ei;
        // lane k forms F[k][j] for j = k+2 .. 4; lane 0 also the G_i
        float pr = er, pi = ei;
        if (k == 0) {
            fr[gslot(1) * NP] = pr;
            fi[gslot(1) * NP] = -pi;
        }
#pragma unroll
        for (int j2 = 2; j2 <= 4; ++j2) {
            const int jj = k + j2;
            if (jj > 4) break;
            float nr_, ni_;
            cmul(pr, pi, Er[jj - 1], Ei[jj - 1], nr_, ni_);
            pr = nr_;
            pi = ni_;
            fr[fslot(k, jj) * NP] = pr;
            fi[fslot(k, jj) * NP] = pi;
            if (k == 0 && jj < 4) {
                fr[gslot(jj) * NP] = pr;
                fi[gslot(jj) * NP] = -pi;
            }
        }
    }
    __syncthreads();
}

// Decay rate (times log2 e) and rotation frequency of mode m = threadIdx.x of
// head h, loaded one chunk ahead; mode_rates_from writes them to F_A2 / F_W.
struct ModePrefetch {
    float alog, w;
};
__device__ __forceinline__ ModePrefetch mode_load(const Params &p, int h) {
    ModePrefetch r{0.f, 0.f};
    const int m = threadIdx.x;
    if (m < p.nr + p.np) {
        r.alog = __ldg(p.A_log + h * p.ndec + (p.per_coord ? m : 0));
        // per-token angles come from F_TH (chunk_angles), not from a frequency
        if (m >= p.nr && !p.angle_tok) r.w = __ldg(p.theta + h * p.np + (m - p.nr));
    }
    return r;
}
__device__ __forceinline__ void mode_rates_from(const Params &p, float *f32, const ModePrefetch &r) {
    const int m = threadIdx.x;
    if (m < NP) {
        const bool on = m < p.nr + p.np;
        f32[F_A2 + m] = on ? -expf(r.alog) * 1.4426950408889634f : 0.f;
        f32[F_W + m] = on ? r.w : 0.f;
    }
}
__device__ __forceinline__ void mode_rates(const Params &p, float *f32, int h) {
    mode_rates_from(p, f32, mode_load(p, h));
}

__device__ __forceinline__ long long bhc(const Params &p, int b, int h, int c) {
    return ((long long)b * p.H + h) * p.nc + c;
}

// ---- chunk states in the operand-tile format ----------------------------------
// The state entering a chunk (and the adjoint carried into it) are stored per
// chunk as 32 KB: the bf16 tile with byte(n, p) = (n/8)*1024 + (p/8)*128 +
// (n%8)*16 + (p%8)*2 for 128 rows x 64 p (rows past N zero), then the tile of
// the bf16 residuals v - hi.  That layout is both K-major with rows n (K = p)
// and MN-major with M or N = p (K = n); consumers bulk-copy it straight into
// their operand tiles.  Before the passes rewrite a slot, it holds the
// chunk-local fp32 sum [N][64].
constexpr int SLOT_FLOATS = NP * PD;            // floats per chunk slot
constexpr uint32_t TILE_BYTES = NP * PD * 2;    // one bf16 tile

__device__ __forceinline__ float2 bf2_to_f2(uint32_t w) {
    return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}

// 8 consecutive p of two state rows n0, n0 + 1 (n0 even): the unit of the
// elementwise passes, moved in 16-byte pieces.
struct Rows2x8 {
    float a[8], d[8];
};
__device__ __forceinline__ void rows_load_f32(const float *slot, int n0, int p8, Rows2x8 &r) {
    const float4 *s0 = reinterpret_cast<const float4 *>(slot + (long long)n0 * PD + p8);
    const float4 *s1 = reinterpret_cast<const float4 *>(slot + (long long)(n0 + 1) * PD + p8);
    const float4 a0 = s0[0], a1 = s0[1], d0 = s1[0], d1 = s1[1];
    r.a[0] = a0.x; r.a[1] = a0.y; r.a[2] = a0.z; r.a[3] = a0.w;
    r.a[4] = a1.x; r.a[5] = a1.y; r.a[6] = a1.z; r.a[7] = a1.w;
    r.d[0] = d0.x; r.d[1] = d0.y; r.d[2] = d0.z; r.d[3] = d0.w;
    r.d[4] = d1.x; r.d[5] = d1.y; r.d[6] = d1.z; r.d[7] = d1.w;
}
// -> hi / lo operand tiles of a chunk slot (row n0 + 1 lies 16 bytes after row n0)
__device__ __forceinline__ void rows_store_tile(unsigned char *slot, int n0, int p8,
                                                const Rows2x8 &r) {
    const uint32_t off = off_kmaj(n0, p8, 128u, 1024u);
    const float *v[2] = {r.a, r.d};
#pragma unroll
    for (int q = 0; q < 2; ++q) {
        float hi[8], lo[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            hi[j] = __bfloat162float(__float2bfloat16_rn(v[q][j]));
            lo[j] = v[q][j] - hi[j];
        }
        st16(slot, off + 16 * q, hi);
        st16(slot + TILE_BYTES, off + 16 * q, lo);
    }
}
__device__ __forceinline__ void rows_load_tile(const unsigned char *slot, int n0, int p8,
                                               Rows2x8 &r) {
    const uint32_t off = off_kmaj(n0, p8, 128u, 1024u);
    float *v[2] = {r.a, r.d};
#pragma unroll
    for (int q = 0; q < 2; ++q) {
        const uint4 h = __ldg(reinterpret_cast<const uint4 *>(slot + off + 16 * q));
        const uint4 l = __ldg(reinterpret_cast<const uint4 *>(slot + TILE_BYTES + off + 16 * q));
        const uint32_t hw[4] = {h.x, h.y, h.z, h.w}, lw[4] = {l.x, l.y, l.z, l.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float2 hh = bf2_to_f2(hw[j]), ll = bf2_to_f2(lw[j]);
            v[q][2 * j] = hh.x + ll.x;
            v[q][2 * j + 1] = hh.y + ll.y;
        }
    }
}

// Work item of the persistent chunk kernels: chunk fastest, then head, then batch row.
struct ChunkItem {
    int c, h, b;
};
__device__ __forceinline__ ChunkItem chunk_item(const Params &p, int item) {
    ChunkItem r;
    r.c = item % p.nc;
    const int rest = item / p.nc;
    r.h = rest % p.H;
    r.b = rest / p.H;
    return r;
}

// ---- chunks chained through a carry in global memory ---------------------------
// A persistent kernel walks the chunks of every (b, h) in order (forward) or in
// reverse (backward), chunk slowest.  The item of the r-th chunk of a (b, h) in
// walking order reads the fp32 carry from slot r & 1 once the counter of
// (b, h) reaches r, writes the next carry to slot (r + 1) & 1 and sets the
// counter to r + 1.
//
// Work items are handed out by a ticket counter in the workspace (zeroed with
// the carry counters on every call): a CTA takes its next item, one ahead of
// the one it works on, with an atomic increment.  Tickets only go to CTAs that
// are running, in increasing order, so the item an item waits on (the same
// (b, h), one chunk earlier in walking order, hence a smaller ticket) is held
// by a running CTA; the smallest unfinished item never waits, so the chain
// always progresses, whatever number of CTAs is resident.
// A carry wait gives up after Params::wait_limit polls; the CTA then raises the
// device error word, sets the call's abort word (so that every other wait of
// the call gives up at once instead of polling to its own limit) and stops.
constexpr long long DEFAULT_WAIT_LIMIT = 1ll << 22;   // polls of a carry counter (~0.5 s)

__device__ __forceinline__ int *chain_ticket(const Params &p) { return p.ws_flag + p.Bsz * p.H; }
__device__ __forceinline__ int *chain_abort_word(const Params &p) {
    return p.ws_flag + p.Bsz * p.H + 1;
}

// Wait until *flag >= target: at most `limit` polls (none for limit 0, which
// makes every wait give up), and none after the call's abort word is set.
__device__ __forceinline__ bool wait_count(const int *flag, int target, const int *abort_word,
                                           long long limit) {
    for (long long i = 0; i < limit; ++i) {
        int v;
        asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(flag) : "memory");
        if (v >= target) return true;
        if ((i & 15) == 15) {
            int a;
            asm volatile("ld.relaxed.gpu.global.b32 %0, [%1];" : "=r"(a) : "l"(abort_word) : "memory");
            if (a) return false;
        }
        __nanosleep(64);
    }
    return false;
}
__device__ __forceinline__ void publish_count(int *flag, int v) {
    __threadfence();
    asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(flag), "r"(v) : "memory");
}
__device__ __forceinline__ void chain_abort(const Params &p) { atomicExch(chain_abort_word(p), 1); }

// Loads (TMA / bulk copies) and MMA commits completing on one mbarrier, counted
// by the issuing thread, so that a CTA that stops early can wait for every
// phase still outstanding before its shared memory and TMEM go away.
struct PhaseCount {
    uint32_t issued, done;
};
// Wait for every outstanding phase (bounded); false if one did not complete.
__device__ __forceinline__ bool drain_phases(uint64_t *bar, PhaseCount &pc) {
    while (pc.done < pc.issued) {
        if (!mbar_wait(bar, pc.done & 1u, WAIT_LIMIT)) return false;
        ++pc.done;
    }
    return true;
}

// item -> (chunk, head, batch row), chunk slowest
__device__ __forceinline__ ChunkItem chunk_item_cs(const Params &p, int item) {
    ChunkItem r;
    const int bh_n = p.Bsz * p.H;
    r.c = item / bh_n;
    const int rest = item - r.c * bh_n;
    r.b = rest / p.H;
    r.h = rest - r.b * p.H;
    return r;
}

// 4 float4 of the carry: thread (row n, column block cq) holds p = 16 cq + 4 j4 + 0..3;
// slot layout [cq][j4][row][4] so that a warp reads 32 consecutive rows.
__device__ __forceinline__ float4 *carry_ptr(const Params &p, int slot, int bh, int cq, int n) {
    return reinterpret_cast<float4 *>(p.ws_ring) +
           (((long long)(slot * p.Bsz * p.H + bh) * 4 + cq) * 4) * NP + n;
}

// item -> (chunk, head, batch row), chunk slowest, last chunk first (the walk of
// the backward, whose carry runs from the end of the sequence)
__device__ __forceinline__ ChunkItem chunk_item_rcs(const Params &p, int item) {
    ChunkItem r = chunk_item_cs(p, item);
    r.c = p.nc - 1 - r.c;
    return r;
}

// ---- host side ---------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    }
    return fn;
}

// 4-D bf16 map over (inner, dim1, time, batch) with a box of (inner, 1, Q, 1).
static bool make_map(CUtensorMap *m, const void *base, uint64_t inner, uint64_t d1, uint64_t L,
                     uint64_t B, uint64_t s1, uint64_t sL, uint64_t sB, uint32_t box_inner,
                     bool swizzle128) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[4] = {inner, d1, L, B};
    cuuint64_t strides[3] = {s1 * 2, sL * 2, sB * 2};
    cuuint32_t box[4] = {box_inner, 1, (cuuint32_t)Q, 1};
    cuuint32_t es[4] = {1, 1, 1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims, strides,
                    box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// Host: calls fn(tok, zoh) with std::integral_constant<bool, ...> arguments for the
// call's angle mode (per-token angles) and write form (ZOH), so that each kernel
// runs the instantiation compiled for them.
template <typename Fn>
static cudaError_t by_variant(const Params &p, Fn &&fn) {
    using T = std::true_type;
    using F = std::false_type;
    if (p.angle_tok) return p.zoh ? fn(T{}, T{}) : fn(T{}, F{});
    return p.zoh ? fn(F{}, T{}) : fn(F{}, F{});
}

}  // namespace chunkc
}  // namespace ssm
