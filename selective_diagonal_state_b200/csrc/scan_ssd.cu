// Chunked tensor-core scan for a per-head (scalar) decay: the Mamba-2 SISO and
// SSD-MIMO configurations ("When a Diagonal State Is Not Enough",
// sungsoo.github.io, Part 03 "Selective SSM and masked linear attention" and
// "SISO and MIMO"; Part 08 item 3), bf16 I/O, fp32 state, head dim 64, 64 or
// 128 state rows, ranks R, O in {1, 2, 4}, optional two-endpoint writes.
//
// With one decay a per head the transition between tokens s < t is the scalar
// exp(a (S_t - S_s)), S the cumulative sum of dt, so the state-mediated part
// of the scan is unnormalised masked linear attention (Thm 24 of Part 03): a
// chunk's output is
//     Y = (C B^T (.) W) X + diag(e) C K_in + D X
// where the rows of X, B (sources) and of Y, C (targets) are the chunk's
// (token, rank) pairs -- R value rows per token, so SSD-MIMO is the SISO form
// with R source and O target rows per token (Part 03 "SISO and MIMO") --,
// W[j, i] = exp(a (S_tj - S_ti)) sigma_ti for t_i < t_j, gamma_tj for
// t_i = t_j and 0 after (the two-endpoint write in the pre-state form
// K_t = A_t K_{t-1} + sigma_t W_t, sigma_t = gamma_t + beta_{t+1}, whose
// readout C_t K_t - beta_{t+1} C_t W_t leaves gamma_t on the diagonal),
// e_t = exp(a S_t) and K_in the state entering the chunk.  The chunk's end
// state is
//     K_out = E K_in + B^T diag(f) X,   f_t = exp(a (S_end - S_t)) sigma_t,
//     E = exp(a S_end).
// Every exponent is <= 0, so no range condition applies.
//
// A chunk has 128 (token, rank) rows: 128 / max(R, O) tokens.  When R != O the
// narrower side's extra rank rows are zero: the tensor maps of x, B (R ranks) and
// of y, C, dy (O ranks) all use a box of max(R, O) ranks, TMA fills the rows past
// a tensor's own rank count with zeros on a load and drops them on a store, so a
// zero source row adds nothing and a zero target row is never written.  Per chunk,
// on the
// tensor cores (M = 128 everywhere, fp32 accumulators in TMEM):
//     CB   = C (128 j x N) . B^T (N x 128 i)
//     S_c  = B^T (N x 128 i) . X' (128 i x 64 p),   X' = diag(f) X
//     Y_d  = P (128 j x 128 i) . X (128 i x 64 p),  P = CB (.) W  (bf16)
//     Y_o  = C (128 j x N) . K_in (N x 64 p)
// and y = Y_d + e Y_o + D x.  k_ssd_fwd is persistent: items are (chunk, head,
// batch row) with the chunk slowest, handed out by a ticket counter; the state
// is carried between the chunks of a (b, h) through two fp32 slots in global
// memory (L2), the same chain as the per-coordinate kernels.
#include <cuda.h>

#include "chunk_common.cuh"
#include "common.cuh"
#include "umma.cuh"

namespace ssm {

// Device word raised by the bounded waits of these kernels (0 = no error).
__device__ int ssm_ssd_error_word;
__device__ __forceinline__ void ssd_raise_error(int code) {
    atomicCAS(&ssm_ssd_error_word, 0, code);
}

namespace ssdk {

using namespace umma;
using namespace chunkc;

constexpr int ROWS = 128;                 // (token, rank) rows per chunk
constexpr int THREADS = 256;              // two CTAs per SM
constexpr uint32_t TILE = 16384;          // 128 rows x 128 bytes (64 bf16), 128-byte swizzle
constexpr uint32_t TMEM_COLS = 256;       // CB 0..127 (then Y_o 0..63) | S_c 128.. | Y_d 192..
constexpr uint32_t SM_X = 0;              // 16 KB x tile (rows (t, r))
constexpr uint32_t SM_B = 16384;          // 2 x 16 KB B (state rows 0-63 | 64-127), rows (t, r);
                                          // then the masked scores P, no-swizzle K-major
constexpr uint32_t SM_C = 49152;          // 2 x 16 KB C, rows (t, o)
constexpr uint32_t SM_XS = 81920;         // 16 KB diag(f) x, then K_in (bf16 [n][p]), then y
constexpr uint32_t SM_F32 = 98304;
// fp32 scratch (float offsets)
constexpr int F_DT = 0;      // [129] dt of the chunk's tokens and of the token after it
constexpr int F_LAM = 132;   // [129] lambda of the same tokens
constexpr int F_S = 264;     // [128] inclusive cumulative sum of dt inside the chunk
constexpr int F_SIG = 392;   // [128] sigma_t = gamma_t + beta_{t+1}
constexpr int F_GAM = 520;   // [128] gamma_t
constexpr int F_FW = 648;    // [128] f_t = e^{a (S_end - S_t)} sigma_t
constexpr int F_EW = 776;    // [128] e_t = e^{a S_t}
constexpr int F_SC = 904;    // [0] a log2(e), [1] D, [2] E = e^{a S_end}
constexpr int F_END = 912;
constexpr uint32_t SM_BAR = SM_F32 + F_END * 4;
constexpr uint32_t SMEM_BYTES = SM_BAR + 128 + 1024;
static_assert(SM_BAR % 8 == 0 && 2 * (SMEM_BYTES + 1024) <= 233472, "two CTAs per SM");

// Tokens of one chunk: dt and lambda (bf16 bits) of tokens t0 .. t0 + Qt, loaded
// one item ahead and converted when stored.
struct Tok {
    unsigned short dv, lv;
};
__device__ __forceinline__ Tok tok_load_q(const Params &p, int b, int h, int t0, int Qt) {
    Tok r{0, 0x3f80};   // dt 0 (tokens past L add nothing), lambda 1
    const int i = threadIdx.x, t = t0 + i;
    if (i <= Qt && t < p.L) {
        r.dv = __ldg(reinterpret_cast<const unsigned short *>(p.dt) + ix_dt(p, b, t, h));
        if (p.two_ep)
            r.lv = __ldg(reinterpret_cast<const unsigned short *>(p.lam) + ix_lam(p, b, t, h));
    }
    return r;
}

// Per-token quantities of the chunk (S, sigma, gamma, f, e) and E, from the
// prefetched dt / lambda; contains barriers (all threads).
__device__ __forceinline__ void chunk_scalars(const Params &p, float *f32, int t0, int Qt,
                                              const Tok &r, float alog, float *fe = nullptr) {
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid <= Qt) {
        f32[F_DT + tid] = __uint_as_float((uint32_t)r.dv << 16);
        f32[F_LAM + tid] = __uint_as_float((uint32_t)r.lv << 16);
    }
    if (tid == 0) f32[F_SC] = -expf(alog) * 1.4426950408889634f;
    __syncthreads();
    if (warp == 0) {
        // inclusive prefix of dt: lane l takes tokens [l * per, (l + 1) * per)
        const int per = Qt >> 5;
        float loc[4];
        float run = 0.f;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            if (k < per) run += f32[F_DT + lane * per + k];
            loc[k] = run;
        }
        float v = run;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float u = __shfl_up_sync(0xffffffffu, v, o);
            if (lane >= o) v += u;
        }
        const float base = v - run;
#pragma unroll
        for (int k = 0; k < 4; ++k)
            if (k < per) f32[F_S + lane * per + k] = base + loc[k];
    } else if (tid >= 32 && tid < 32 + Qt) {
        const int t = tid - 32;
        const float dv = f32[F_DT + t], lv = f32[F_LAM + t];
        const float bn = (t0 + t + 1 < p.L) ? (1.f - f32[F_LAM + t + 1]) * f32[F_DT + t + 1] : 0.f;
        const float g = lv * dv;
        f32[F_GAM + t] = g;
        f32[F_SIG + t] = g + bn;
    }
    __syncthreads();
    if (tid < Qt) {
        const float a2 = f32[F_SC], se = f32[F_S + Qt - 1], st = f32[F_S + tid];
        const float dend = ex2_fast(a2 * (se - st));
        f32[F_FW + tid] = dend * f32[F_SIG + tid];
        f32[F_EW + tid] = ex2_fast(a2 * st);
        if (fe) fe[tid] = dend;
        if (tid == 0) f32[F_SC + 2] = ex2_fast(a2 * se);
    }
    __syncthreads();
}

// 8 bf16 of row `row`, logical 16-byte chunk `lc` of a 128-byte-swizzled tile
__device__ __forceinline__ uint32_t sw_off(int row, int lc) {
    return (uint32_t)row * 128u + ((uint32_t)(lc ^ (row & 7)) << 4);
}
__device__ __forceinline__ void unpack8(const uint4 w, float (&v)[8]) {
    const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        v[2 * i] = __uint_as_float(u[i] << 16);
        v[2 * i + 1] = __uint_as_float(u[i] & 0xffff0000u);
    }
}
__device__ __forceinline__ uint4 pack8(const float (&v)[8]) {
    uint4 w;
    w.x = pack_bf16(v[0], v[1]);
    w.y = pack_bf16(v[2], v[3]);
    w.z = pack_bf16(v[4], v[5]);
    w.w = pack_bf16(v[6], v[7]);
    return w;
}

// ---- segments -----------------------------------------------------------------
// The forward advances the state of a (b, h) a segment of G chunks at a time.  With
// one decay per head the state a segment adds is one contraction over all its rows,
//     S_seg = B_seg^T diag(e^{a (S_end - S_t)} sigma_t) X_seg,   E_seg = e^{a S_end}
// (S the sum of dt inside the segment), the chunk state over a longer span: the
// states entering the segments then come from a short elementwise pass over the
// segments, and the forward's work items - whole segments, walked chunk by chunk
// with the carry kept by the CTA - wait on no other item.
// Slots as the carry: [segment][b * H + h][cq][j4][n][4] fp32.
__device__ __forceinline__ float4 *seg_ptr(const Params &p, int s, int bh, int cq, int n) {
    return reinterpret_cast<float4 *>(p.sd_seg) +
           (((long long)(s * p.Bsz * p.H + bh) * 4 + cq) * 4) * NP + n;
}
__device__ __forceinline__ float4 *priv_ptr(const Params &p, int cta, int cq, int n) {
    return reinterpret_cast<float4 *>(p.sd_priv) + (((long long)cta * 4 + cq) * 4) * NP + n;
}
__device__ __forceinline__ void ld_slot16(const float4 *src, float (&v)[16]) {
#pragma unroll
    for (int j4 = 0; j4 < 4; ++j4) {
        const float4 w = __ldcg(src + j4 * NP);
        v[4 * j4] = w.x;
        v[4 * j4 + 1] = w.y;
        v[4 * j4 + 2] = w.z;
        v[4 * j4 + 3] = w.w;
    }
}
__device__ __forceinline__ void st_slot16(float4 *dst, const float (&v)[16]) {
#pragma unroll
    for (int j4 = 0; j4 < 4; ++j4)
        __stcg(dst + j4 * NP, make_float4(v[4 * j4], v[4 * j4 + 1], v[4 * j4 + 2], v[4 * j4 + 3]));
}

// S_seg and E_seg of every (segment, b, h): the segment's chunks last to first, the
// contraction accumulated in TMEM, each chunk's f_t scaled by the decay of the chunks
// after it.  Work items are independent (no chain).
__global__ void __launch_bounds__(THREADS, 2)
k_ssd_seg_state(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmB,
                Params p, int lgR) {
    const int BH = p.Bsz * p.H, G = p.sd_G;
    const int nitems = p.sd_nseg * BH;
    if ((int)blockIdx.x >= nitems) return;
    extern __shared__ unsigned char smem_raw[];
    unsigned char *sm = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    float *f32 = reinterpret_cast<float *>(sm + SM_F32);
    uint64_t *bar_in = reinterpret_cast<uint64_t *>(sm + SM_BAR);   // x and B of a chunk
    uint64_t *bar_mma = bar_in + 1;
    uint32_t *tslot = reinterpret_cast<uint32_t *>(bar_in + 2);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int N = p.N, nbox = N / 64, Qt = ROWS >> lgR;
    const int qd = warp & 3, cb2 = warp >> 2, row = 32 * qd + lane;
    PhaseCount pc_in = {0u, 0u}, pc_m = {0u, 0u};   // issued: thread 0; done: every thread
    if (tid == 0) {
        mbar_init(bar_in, 1);
        mbar_init(bar_mma, 1);
        mbar_fence_init();
        tma_prefetch_desc(&tmX);
        tma_prefetch_desc(&tmB);
    }
    if (warp == 0) tmem_alloc(tslot, 64);
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t t_s = *tslot, lane_q = (32u * qd) << 16;
    bool aborted = false;
    for (int item = blockIdx.x; item < nitems && !aborted; item += gridDim.x) {
        const int sg = item / BH, bh = item - sg * BH, b = bh / p.H, h = bh - b * p.H;
        const int c0 = sg * G, glen = min(G, p.nc - c0);
        const float alog = __ldg(p.A_log + h * p.ndec);
        float P = 1.f;   // decay of the segment's chunks after the current one
        for (int jj = glen - 1; jj >= 0; --jj) {
            const int c = c0 + jj, t0 = c * Qt;
            if (tid == 0) {
                mbar_expect_tx(bar_in, TILE * (1 + nbox));
                tma_load_5d(sm + SM_X, &tmX, bar_in, 0, 0, h, t0, b);
                for (int k = 0; k < nbox; ++k)
                    tma_load_5d(sm + SM_B + k * TILE, &tmB, bar_in, 64 * k, 0, h / p.hpg, t0, b);
                ++pc_in.issued;
            }
            const Tok tok = tok_load_q(p, b, h, t0, Qt);
            chunk_scalars(p, f32, t0, Qt, tok, alog);
            int ok = mbar_wait(bar_in, pc_in.done & 1u, WAIT_LIMIT) ? 1 : 0;
            pc_in.done += (uint32_t)ok;
            if (!ok) ssd_raise_error(1);
            if (!__syncthreads_and(ok)) {
                aborted = true;
                break;
            }
            // X' = diag(f P) X
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int ch = tid + THREADS * q;
                const int r = ch >> 3;
                const uint32_t off = (uint32_t)r * 128u + (uint32_t)(ch & 7) * 16u;
                const float f = f32[F_FW + (r >> lgR)] * P;
                float v[8];
                unpack8(*reinterpret_cast<const uint4 *>(sm + SM_X + off), v);
#pragma unroll
                for (int j = 0; j < 8; ++j) v[j] *= f;
                *reinterpret_cast<uint4 *>(sm + SM_XS + off) = pack8(v);
            }
            fence_proxy_async();
            fence_before_sync();
            __syncthreads();
            if (tid == 0) {
                fence_after_sync();
                const uint32_t b_base = smem_u32(sm + SM_B), xs_base = smem_u32(sm + SM_XS);
                const uint32_t id = idesc_bf16(128, 64, true, true);
                for (int s2 = 0; s2 < ROWS / 16; ++s2)
                    mma_bf16(t_s, sdesc(b_base + s2 * 2048u, TILE, 1024u, LAYOUT_SW128),
                             sdesc(xs_base + s2 * 2048u, TILE, 1024u, LAYOUT_SW128), id,
                             s2 > 0 || jj < glen - 1);
                mma_commit(bar_mma);
                ++pc_m.issued;
            }
            ok = mbar_wait(bar_mma, pc_m.done & 1u, WAIT_LIMIT) ? 1 : 0;
            pc_m.done += (uint32_t)ok;
            if (!ok) ssd_raise_error(1);
            fence_after_sync();
            P *= f32[F_SC + 2];
            if (!__syncthreads_and(ok)) {   // also: every thread has read this chunk's scalars
                aborted = true;
                break;
            }
        }
        if (aborted) break;
#pragma unroll
        for (int q = 0; q < 2; ++q) {
            const int cq = 2 * cb2 + q;
            float v[16];
            tmem_ld16(t_s + lane_q + 16u * cq, v);
            if (row >= N)
#pragma unroll
                for (int j = 0; j < 16; ++j) v[j] = 0.f;
            st_slot16(seg_ptr(p, sg, bh, cq, row), v);
        }
        if (tid == 0) p.sd_sege[(long long)sg * BH + bh] = P;
        fence_before_sync();
        __syncthreads();   // TMEM is read before the next item's first MMA overwrites it
        fence_after_sync();
    }
    if (aborted && tid == 0) {
        drain_phases(bar_in, pc_in);
        drain_phases(bar_mma, pc_m);
    }
    fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        fence_after_sync();
        tmem_dealloc(t_s, 64);
    }
}

// The state entering every segment of a (b, h), in place of S_seg: thread (row n,
// column block cq, 4 columns j4) of (b, h) = blockIdx.y, segments in order, the
// loads of the next PF segments in flight while the current one is carried.
constexpr int SEG_PF = 4;
__global__ void __launch_bounds__(256) k_ssd_seg_pass(Params p) {
    const int bh = blockIdx.y, b = bh / p.H, h = bh - b * p.H, BH = p.Bsz * p.H;
    const int e = blockIdx.x * 256 + threadIdx.x;   // 0 .. 2047: (cq, j4, n)
    const int n = e & 127, j4 = (e >> 7) & 3, cq = e >> 9;
    float4 K = make_float4(0.f, 0.f, 0.f, 0.f);
    if (n < p.N) {
        float beta0 = 0.f;
        if (p.two_ep)
            beta0 = (1.f - ld_io(p.lam, ix_lam(p, b, 0, h), 1)) * ld_io(p.dt, ix_dt(p, b, 0, h), 1);
        float v[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const long long i0 = ix_st(p, b, h, n, 16 * cq + 4 * j4 + k);
            v[k] = p.h0 ? p.h0[i0] : 0.f;
            if (p.w0) v[k] = fmaf(beta0, p.w0[i0], v[k]);
        }
        K = make_float4(v[0], v[1], v[2], v[3]);
    }
    const int ns = p.sd_nseg;
    float4 buf[SEG_PF];
    float eb[SEG_PF];
#pragma unroll
    for (int k = 0; k < SEG_PF; ++k) {
        if (k < ns) {
            buf[k] = __ldcg(seg_ptr(p, k, bh, cq, n) + j4 * NP);
            eb[k] = p.sd_sege[(long long)k * BH + bh];
        }
    }
    for (int s0 = 0; s0 < ns; s0 += SEG_PF) {
#pragma unroll
        for (int k = 0; k < SEG_PF; ++k) {
            const int sg = s0 + k;
            if (sg < ns) {
                const float4 sv = buf[k];
                const float E = eb[k];
                if (sg + SEG_PF < ns) {   // refill this stage with a later segment
                    buf[k] = __ldcg(seg_ptr(p, sg + SEG_PF, bh, cq, n) + j4 * NP);
                    eb[k] = p.sd_sege[(long long)(sg + SEG_PF) * BH + bh];
                }
                __stcg(seg_ptr(p, sg, bh, cq, n) + j4 * NP, K);
                K = make_float4(fmaf(E, K.x, sv.x), fmaf(E, K.y, sv.y), fmaf(E, K.z, sv.z),
                                fmaf(E, K.w, sv.w));
            }
        }
    }
}

__global__ void __launch_bounds__(THREADS, 2)
k_ssd_fwd(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmB,
          const __grid_constant__ CUtensorMap tmC, const __grid_constant__ CUtensorMap tmY,
          Params p, int lgR) {
    const int BH = p.Bsz * p.H, G = p.sd_G;
    const int nitems = p.nc * BH;            // chunk items (c * BH + bh); nitems = none
    const int nseg_items = p.sd_nseg * BH;   // tickets: (segment, b, h), segment slowest
    if ((int)blockIdx.x >= nseg_items) return;
    extern __shared__ unsigned char smem_raw[];
    unsigned char *sm = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    float *f32 = reinterpret_cast<float *>(sm + SM_F32);
    uint64_t *bar_x = reinterpret_cast<uint64_t *>(sm + SM_BAR);   // x tile
    uint64_t *bar_b = bar_x + 1, *bar_c = bar_x + 2;               // B, C tiles
    uint64_t *bar_sc = bar_x + 3, *bar_y = bar_x + 4;              // MMA phases
    uint32_t *tslot = reinterpret_cast<uint32_t *>(bar_x + 5);
    int *s_item = reinterpret_cast<int *>(bar_x + 6);               // [2] claimed tickets

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int N = p.N, L = p.L;
    const int nbox = N / 64;
    const int Qt = ROWS >> lgR;   // tokens per chunk
    const bool want_y = p.y != nullptr;
    const int qd = warp & 3, cb2 = warp >> 2;   // TMEM lane quarter, column half
    const int row = 32 * qd + lane;             // TMEM lane = row of every M = 128 tile
    unsigned char *sX = sm + SM_X;

    auto issue_x = [&](int item) {
        const ChunkItem it = chunk_item_cs(p, item);
        mbar_expect_tx(bar_x, TILE);
        tma_load_5d(sX, &tmX, bar_x, 0, 0, it.h, it.c * Qt, it.b);
    };
    auto issue_b = [&](int item) {
        const ChunkItem it = chunk_item_cs(p, item);
        mbar_expect_tx(bar_b, TILE * nbox);
        for (int k = 0; k < nbox; ++k)
            tma_load_5d(sm + SM_B + k * TILE, &tmB, bar_b, 64 * k, 0, it.h / p.hpg, it.c * Qt, it.b);
    };
    auto issue_c = [&](int item) {
        const ChunkItem it = chunk_item_cs(p, item);
        mbar_expect_tx(bar_c, TILE * nbox);
        for (int k = 0; k < nbox; ++k)
            tma_load_5d(sm + SM_C + k * TILE, &tmC, bar_c, 64 * k, 0, it.h / p.hpg, it.c * Qt, it.b);
    };

    PhaseCount pc_x = {0u, 0u}, pc_b = {0u, 0u}, pc_c = {0u, 0u};
    PhaseCount pc_sc = {0u, 0u}, pc_y = {0u, 0u};
    if (tid == 0) {
        for (int i = 0; i < 5; ++i) mbar_init(&bar_x[i], 1);
        mbar_fence_init();
        tma_prefetch_desc(&tmX);
        tma_prefetch_desc(&tmB);
        tma_prefetch_desc(&tmC);
        if (want_y) tma_prefetch_desc(&tmY);
        // < nseg_items: the grid is <= nseg_items
        const int first = atomicAdd(chain_ticket(p), 1);
        s_item[0] = first;
        const int fitem = (first / BH) * G * BH + first % BH;   // its first chunk
        issue_x(fitem);
        ++pc_x.issued;
        issue_b(fitem);
        ++pc_b.issued;
        if (want_y) {   // C is read by the outputs only
            issue_c(fitem);
            ++pc_c.issued;
        }
    }
    if (warp == 0) tmem_alloc(tslot, TMEM_COLS);
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tbase = *tslot;
    const uint32_t t_cb = tbase, t_yo = tbase, t_sc = tbase + 128u, t_yd = tbase + 192u;
    const uint32_t lane_q = (32u * qd) << 16;
    int tk = s_item[0], jj = 0;   // segment ticket, chunk inside the segment
    int item = (tk / BH) * G * BH + tk % BH;
    Tok tok;
    float alog;
    {
        const ChunkItem it = chunk_item_cs(p, item);
        tok = tok_load_q(p, it.b, it.h, it.c * Qt, Qt);
        alog = __ldg(p.A_log + it.h * p.ndec);
    }
    bool aborted = false;

    for (int k = 0; item < nitems; ++k) {
        // the segment after this one, claimed at its first chunk
        if (tid == 0 && jj == 0) s_item[1] = atomicAdd(chain_ticket(p), 1);
        const uint32_t par = (uint32_t)(k & 1);
        const ChunkItem it = chunk_item_cs(p, item);
        const int c = it.c, h = it.h, b = it.b;
        const int bh = b * p.H + h;
        const int t0 = c * Qt;
        const int sg = tk / BH, glen = min(G, p.nc - sg * G);
        // the previous item's y store has read the staging tile
        if (tid == 0) bulk_wait_read_all();
        chunk_scalars(p, f32, t0, Qt, tok, alog);
        // the next chunk: the segment's next, or the first of the next claimed segment
        const int ntk = jj + 1 < glen ? tk : s_item[1];
        const int njj = jj + 1 < glen ? jj + 1 : 0;
        const int next = ntk < nseg_items ? ((ntk / BH) * G + njj) * BH + ntk % BH : nitems;
        if (next < nitems) {
            const ChunkItem nx = chunk_item_cs(p, next);
            tok = tok_load_q(p, nx.b, nx.h, nx.c * Qt, Qt);
            alog = __ldg(p.A_log + nx.h * p.ndec);
            if (tid == 0) {   // the next item's tiles stream into L2 while this one runs
                const int g2 = nx.h / p.hpg;
                tma_prefetch_5d(&tmX, 0, 0, nx.h, nx.c * Qt, nx.b);
                for (int kb = 0; kb < nbox; ++kb) {
                    tma_prefetch_5d(&tmB, 64 * kb, 0, g2, nx.c * Qt, nx.b);
                    if (want_y) tma_prefetch_5d(&tmC, 64 * kb, 0, g2, nx.c * Qt, nx.b);
                }
            }
        }
        {
            const bool okx = mbar_wait(bar_x, par, WAIT_LIMIT);
            const bool okb = okx && mbar_wait(bar_b, par, WAIT_LIMIT);
            const bool okc = okb && (!want_y || mbar_wait(bar_c, par, WAIT_LIMIT));
            if (tid == 0) {
                pc_x.done += okx ? 1u : 0u;
                pc_b.done += okb ? 1u : 0u;
                pc_c.done += (want_y && okc) ? 1u : 0u;
            }
            int ok = okc ? 1 : 0;
            if (!ok) {
                ssd_raise_error(1);
                chain_abort(p);
            }
            if (!__syncthreads_and(ok)) {
                aborted = true;
                break;
            }
        }
        // ---- CB = C B^T (completion tracked by the S_c commit, which covers it) -----
        if (tid == 0 && want_y) {
            fence_after_sync();
            const uint32_t b_base = smem_u32(sm + SM_B), c_base = smem_u32(sm + SM_C);
            const uint32_t id = idesc_bf16(128, 128, false, false);
            for (int s = 0; s < N / 16; ++s) {
                const uint32_t off = (uint32_t)(s >> 2) * TILE + (uint32_t)(s & 3) * 32u;
                mma_bf16(t_cb, sdesc(c_base + off, 16u, 1024u, LAYOUT_SW128),
                         sdesc(b_base + off, 16u, 1024u, LAYOUT_SW128), id, s > 0);
            }
        }
        // ---- X' = diag(f) X (same swizzled positions) -------------------------------
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int ch = tid + THREADS * q;    // 16-byte chunk: row ch >> 3, position ch & 7
            const int r = ch >> 3;
            const uint32_t off = (uint32_t)r * 128u + (uint32_t)(ch & 7) * 16u;
            const float f = f32[F_FW + (r >> lgR)];
            float v[8];
            unpack8(*reinterpret_cast<const uint4 *>(sX + off), v);
#pragma unroll
            for (int j = 0; j < 8; ++j) v[j] *= f;
            *reinterpret_cast<uint4 *>(sm + SM_XS + off) = pack8(v);
        }
        fence_proxy_async();
        fence_before_sync();
        __syncthreads();
        // ---- S_c = B^T X' (A = B read MN-major over both 64-row halves) ----------------
        if (tid == 0) {
            fence_after_sync();
            const uint32_t b_base = smem_u32(sm + SM_B), xs_base = smem_u32(sm + SM_XS);
            const uint32_t id = idesc_bf16(128, 64, true, true);
            for (int s = 0; s < ROWS / 16; ++s)
                mma_bf16(t_sc, sdesc(b_base + s * 2048u, TILE, 1024u, LAYOUT_SW128),
                         sdesc(xs_base + s * 2048u, TILE, 1024u, LAYOUT_SW128), id, s > 0);
            mma_commit(bar_sc);
            ++pc_sc.issued;
        }
        // ---- chain: K_out = E K_in + S_c -------------------------------------------
        {
            int ok = mbar_wait(bar_sc, par, WAIT_LIMIT) ? 1 : 0;
            if (tid == 0) pc_sc.done += (uint32_t)ok;
            if (!ok) {
                ssd_raise_error(1);
                chain_abort(p);
            }
            fence_after_sync();
            if (!__syncthreads_and(ok)) {
                aborted = true;
                break;
            }
        }
        // states only: B is consumed (CB is not issued): fetch the next item's
        if (!want_y && tid == 0 && next < nitems) {
            issue_b(next);
            ++pc_b.issued;
        }
#pragma unroll 1
        for (int cq = 2 * cb2; cq < 2 * cb2 + 2; ++cq) {
            // K_in as the bf16 tile of the readout, in X''s place (S_c has read X')
            const int n = row;
            // K_in: the state entering the segment (segment pass), then the CTA's own carry
            float kc[16], sc[16];
            ld_slot16(jj == 0 ? seg_ptr(p, sg, bh, cq, n) : priv_ptr(p, blockIdx.x, cq, n), kc);
            tmem_ld16(t_sc + lane_q + 16u * cq, sc);
            const float E = f32[F_SC + 2];
            unsigned char *sv = p.ws_kp
                ? reinterpret_cast<unsigned char *>(p.ws_kp + bhc(p, b, h, c) * SLOT_FLOATS)
                : nullptr;
#pragma unroll
            for (int g8 = 0; g8 < 2; ++g8) {
                float hi[8], lo[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const float v = kc[8 * g8 + j];
                    hi[j] = __bfloat162float(__float2bfloat16_rn(v));
                    lo[j] = v - hi[j];
                }
                const uint32_t off = sw_off(n, 2 * cq + g8);
                const uint4 wh = pack8(hi);
                *reinterpret_cast<uint4 *>(sm + SM_XS + off) = wh;
                if (sv) {
                    *reinterpret_cast<uint4 *>(sv + off) = wh;
                    *reinterpret_cast<uint4 *>(sv + TILE + off) = pack8(lo);
                }
            }
            float kn[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) kn[j] = n < N ? fmaf(E, kc[j], sc[j]) : 0.f;
            if (c + 1 < p.nc) {
                if (jj + 1 < glen) st_slot16(priv_ptr(p, blockIdx.x, cq, n), kn);
            } else if (n < N) {
                // final state (beta_L = 0, so K_{L-1} = H_{L-1}) and the last write
                // W_{L-1} = B_{L-1} u_{L-1} (summed over the R value rows)
                const int g = h / p.hpg, tl = L - 1;
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const long long i0 = ix_st(p, b, h, n, 16 * cq + j);
                    if (p.hT) p.hT[i0] = kn[j];
                    if (p.wT) {
                        float w = 0.f;
                        for (int r = 0; r < p.R; ++r)
                            w = fmaf(ld_io(p.Bm, ix_B(p, b, tl, g, r, n), 1),
                                     ld_io(p.x, ix_x(p, b, tl, h, r, 16 * cq + j), 1), w);
                        p.wT[i0] = w;
                    }
                }
            }
        }
        fence_proxy_async();
        fence_before_sync();
        __syncthreads();
        if (want_y) {
            // ---- masked scores P = CB (.) W -> bf16 tile in B's place (CB and S_c have
            // read B; CB completed with S_c) -------------------------------------------------
#pragma unroll 1
            for (int sub = 0; sub < 2; ++sub) {
                const int i0 = 64 * cb2 + 32 * sub;
                float v[32];
                tmem_ld16(t_cb + lane_q + (uint32_t)i0, *reinterpret_cast<float(*)[16]>(v));
                tmem_ld16(t_cb + lane_q + (uint32_t)i0 + 16u, *reinterpret_cast<float(*)[16]>(v + 16));
                const int tj = row >> lgR;
                const float a2 = f32[F_SC], stj = f32[F_S + tj], gj = f32[F_GAM + tj];
#pragma unroll
                for (int q8 = 0; q8 < 4; ++q8) {
                    float w8[8];
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const int ti = (i0 + 8 * q8 + j) >> lgR;
                        float wt = 0.f;
                        if (ti < tj)
                            wt = ex2_fast(a2 * (stj - f32[F_S + ti])) * f32[F_SIG + ti];
                        else if (ti == tj)
                            wt = gj;
                        w8[j] = v[8 * q8 + j] * wt;
                    }
                    *reinterpret_cast<uint4 *>(sm + SM_B + off_kmaj(row, i0 + 8 * q8, 128u, 2048u)) =
                        pack8(w8);
                }
            }
            fence_proxy_async();
            fence_before_sync();
            __syncthreads();
            // ---- Y_d = P X, Y_o = C K_in ------------------------------------------------
            if (tid == 0) {
                fence_after_sync();
                const uint32_t p_base = smem_u32(sm + SM_B), x_base = smem_u32(sX);
                const uint32_t id = idesc_bf16(128, 64, false, true);
                for (int s = 0; s < ROWS / 16; ++s)
                    mma_bf16(t_yd, sdesc(p_base + s * 256u, 128u, 2048u, LAYOUT_NONE),
                             sdesc(x_base + s * 2048u, TILE, 1024u, LAYOUT_SW128), id, s > 0);
                const uint32_t c_base = smem_u32(sm + SM_C), k_base = smem_u32(sm + SM_XS);
                for (int s = 0; s < N / 16; ++s)
                    mma_bf16(t_yo,
                             sdesc(c_base + (uint32_t)(s >> 2) * TILE + (uint32_t)(s & 3) * 32u,
                                   16u, 1024u, LAYOUT_SW128),
                             sdesc(k_base + s * 2048u, TILE, 1024u, LAYOUT_SW128), id, s > 0);
                mma_commit(bar_y);
                ++pc_y.issued;
            }
            {
                int ok = mbar_wait(bar_y, par, WAIT_LIMIT) ? 1 : 0;
                if (tid == 0) pc_y.done += (uint32_t)ok;
                if (!ok) {
                    ssd_raise_error(1);
                    chain_abort(p);
                }
                fence_after_sync();
                if (!__syncthreads_and(ok)) {
                    aborted = true;
                    break;
                }
            }
            // P (in B's place), C and K_in are consumed: fetch the next item's B and C
            if (tid == 0 && next < nitems) {
                issue_b(next);
                ++pc_b.issued;
                issue_c(next);
                ++pc_c.issued;
            }
            // ---- epilogue: y into K_in's place ------------------------------------------
#pragma unroll 1
            for (int cq = 2 * cb2; cq < 2 * cb2 + 2; ++cq) {
                float yd[16], yo[16];
                tmem_ld16(t_yd + lane_q + 16u * cq, yd);
                tmem_ld16(t_yo + lane_q + 16u * cq, yo);
                const float e = f32[F_EW + (row >> lgR)];
                const float D = (p.R == p.O && p.D) ? __ldg(p.D + h) : 0.f;
#pragma unroll
                for (int g8 = 0; g8 < 2; ++g8) {
                    const uint32_t off = sw_off(row, 2 * cq + g8);
                    float xv[8], yv[8];
                    unpack8(*reinterpret_cast<const uint4 *>(sX + off), xv);
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        yv[j] = fmaf(D, xv[j], fmaf(e, yo[8 * g8 + j], yd[8 * g8 + j]));
                    *reinterpret_cast<uint4 *>(sm + SM_XS + off) = pack8(yv);
                }
            }
            fence_proxy_async();
            fence_before_sync();
            __syncthreads();
            if (tid == 0) {   // rows past the sequence end are clipped by the store
                tma_store_5d(&tmY, sm + SM_XS, 0, 0, h, t0, b);
                bulk_commit();
            }
        }
        fence_before_sync();
        __syncthreads();
        // x is consumed: fetch the next item's
        if (tid == 0 && next < nitems) {
            issue_x(next);
            ++pc_x.issued;
        }
        item = next;
        tk = ntk;
        jj = njj;
    }
    if (tid == 0) bulk_wait_read_all();
    if (aborted && tid == 0) {
        drain_phases(bar_x, pc_x);
        drain_phases(bar_b, pc_b);
        drain_phases(bar_c, pc_c);
        drain_phases(bar_sc, pc_sc);
        drain_phases(bar_y, pc_y);
    }
    fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        fence_after_sync();
        tmem_dealloc(tbase, TMEM_COLS);
    }
}

}  // namespace ssdk

// ============================================================================
// k_ssd_bwd: reverse-mode of one chunk per work item, chunks of a (b, h) walked
// last to first and chained through the adjoint G = dL/dK carried between them
// (two fp32 slots in L2, the same chain as the forward).  With dS = dY X^T,
// w the mask weights and G_out the adjoint of the chunk's end state:
//     dX  = P^T dY + diag(f) B G_out + D dY
//     dB  = (dS (.) W)^T C + diag(f) X G_out^T
//     dC  = (dS (.) W) B + diag(e) dY K_in^T
//     G_in = E G_out + C^T diag(e) dY
// and the gradient of the log-decay rho_u = a dt_u of token u is, exactly,
// the sum over the (write, read) pairs that step u lies between:
//     drho_u = sum_{t_i < u <= t_j} Z[j, i]              (Z = dS (.) CB (.) W)
//            + sum_{t_j >= u} R[j] + sum_{t_i < u} F[i] + Q
// with R[j] = <dY_j, e_j (C K_in)_j> (the entering state read in the chunk),
// F[i] = f_i <X_i, (B G_out)_i> (writes read after the chunk) and
// Q = <G_out, E K_in> (the entering state read after the chunk).  dsigma_t and
// the gamma_t part of the diagonal go to a per-token workspace for the
// token pass (k_ssd_tokens).  Tensor cores (M = 128):
//   phase 1: CB = C B^T, dS = dY X^T, dC <- diag(e) dY K_in^T, G_loc = C^T diag(e) dY
//   phase 2: dX_d = P^T dY, dC += (dS (.) W) B, dB = (dS (.) W)^T C
//   phase 3 (after the chain step): dX_s = B G_out, dB += diag(f) X G_out^T
// ============================================================================
namespace ssdb {
using ssdk::F_DT;
using ssdk::F_EW;
using ssdk::F_FW;
using ssdk::F_GAM;
using ssdk::F_LAM;
using ssdk::F_S;
using ssdk::F_SC;
using ssdk::F_SIG;
using ssdk::ROWS;
using ssdk::TILE;

constexpr int THREADS = 512;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t T_CB = 0, T_DB = 0;       // CB, then dB (128 columns)
constexpr uint32_t T_DS = 128, T_DXS = 128;  // dS, then dX_s (64)
constexpr uint32_t T_DC = 256;               // diag(e) dY K_in^T, then dC (128)
constexpr uint32_t T_GL = 384;               // G_loc (64), read by the chain step
constexpr uint32_t T_BS0 = 192, T_BS1 = 384;  // X G_out^T, state rows 0-63 | 64-127 (phase 3)
constexpr uint32_t T_DXD = 448, T_YO = 448;  // Y_o = C K_in (read by the masking), then dX_d (64)
constexpr uint32_t SM_X = 0;         // 16 KB x (rows (t, r))
constexpr uint32_t SM_DY = 16384;    // 16 KB dy (rows (t, o))
constexpr uint32_t SM_B = 32768;     // 2 x 16 KB B
constexpr uint32_t SM_C = 65536;     // 2 x 16 KB C
constexpr uint32_t SM_K = 98304;     // 16 KB K_in (bf16 hi tile [n][p])
constexpr uint32_t SM_P = 114688;    // 32 KB P; then diag(f) X (16 KB) + G_out [n][p] (16 KB); then dB
constexpr uint32_t SM_DCB = 147456;  // 32 KB dS (.) W; then dC
constexpr uint32_t SM_DYS = 180224;  // 16 KB diag(e) dy, then dx
constexpr uint32_t SM_F32 = 196608;
constexpr int F_FE = 912;            // [128] e^{a (S_end - S_t)}
constexpr int F_RED = 1040;          // [6][4][128] partial row / column sums
constexpr int R_ROWZ = 0, R_DIAG = 512, R_ROFF = 1024, R_COLZ = 1536, R_WQ = 2048, R_DD = 2560;
constexpr int F_QB = F_RED + 3072;   // [16] per-warp partials of Q, then [16] of dbeta_0
constexpr int F_END = F_QB + 32;
constexpr uint32_t SM_BAR = SM_F32 + F_END * 4;
constexpr uint32_t SMEM_BYTES = SM_BAR + 128 + 1024;
static_assert(SM_BAR % 8 == 0 && SMEM_BYTES <= 232448, "shared memory map");
}  // namespace ssdb

__global__ void __launch_bounds__(ssdb::THREADS, 1)
k_ssd_bwd(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmDY,
          const __grid_constant__ CUtensorMap tmB, const __grid_constant__ CUtensorMap tmC,
          const __grid_constant__ CUtensorMap tmDX, const __grid_constant__ CUtensorMap tmDB,
          const __grid_constant__ CUtensorMap tmDC, Params p, int lgR) {
    using namespace ssdb;
    using namespace umma;
    using chunkc::bhc;
    using chunkc::carry_ptr;
    using chunkc::chain_abort;
    using chunkc::chain_abort_word;
    using chunkc::chain_ticket;
    using chunkc::ChunkItem;
    using chunkc::chunk_item_rcs;
    using chunkc::drain_phases;
    using chunkc::ex2_fast;
    using chunkc::NP;
    using chunkc::PhaseCount;
    using chunkc::publish_count;
    using chunkc::SLOT_FLOATS;
    using chunkc::wait_count;
    using chunkc::WAIT_LIMIT;
    using ssdk::pack8;
    using ssdk::sw_off;
    using ssdk::unpack8;
    const int BH = p.Bsz * p.H;
    const int nitems = p.nc * BH;
    if ((int)blockIdx.x >= nitems) return;
    extern __shared__ unsigned char smem_raw[];
    unsigned char *sm = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    float *f32 = reinterpret_cast<float *>(sm + SM_F32);
    float *red = f32 + F_RED;
    uint64_t *bar_x = reinterpret_cast<uint64_t *>(sm + SM_BAR);   // x + dy
    uint64_t *bar_k = bar_x + 1, *bar_bc = bar_x + 2;                 // K_in; B + C
    uint64_t *bar_p1 = bar_x + 3, *bar_p2 = bar_x + 4, *bar_p3 = bar_x + 5;   // MMA phases
    uint32_t *tslot = reinterpret_cast<uint32_t *>(bar_x + 6);
    int *s_item = reinterpret_cast<int *>(bar_x + 7);                // [2] claimed tickets

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int N = p.N, L = p.L;
    const int nbox = N / 64;
    const int Qt = ROWS >> lgR;
    const int Rm = (1 << lgR) - 1;
    const bool one_head = p.hpg == 1;
    const int qd = warp & 3, cb4 = warp >> 2;
    const int row = 32 * qd + lane;
    const uint32_t lane_q = (uint32_t)(32 * qd) << 16;

    auto issue_x = [&](int item) {
        const ChunkItem it = chunk_item_rcs(p, item);
        mbar_expect_tx(bar_x, 2 * TILE);
        tma_load_5d(sm + SM_X, &tmX, bar_x, 0, 0, it.h, it.c * Qt, it.b);
        tma_load_5d(sm + SM_DY, &tmDY, bar_x, 0, 0, it.h, it.c * Qt, it.b);
    };
    auto issue_k = [&](int item) {
        const ChunkItem it = chunk_item_rcs(p, item);
        mbar_expect_tx(bar_k, TILE);
        bulk_load(sm + SM_K, p.ws_kp + bhc(p, it.b, it.h, it.c) * SLOT_FLOATS, TILE, bar_k);
    };
    auto issue_bc = [&](int item) {
        const ChunkItem it = chunk_item_rcs(p, item);
        const int g = it.h / p.hpg;
        mbar_expect_tx(bar_bc, 2 * TILE * nbox);
        for (int k = 0; k < nbox; ++k) {
            tma_load_5d(sm + SM_B + k * TILE, &tmB, bar_bc, 64 * k, 0, g, it.c * Qt, it.b);
            tma_load_5d(sm + SM_C + k * TILE, &tmC, bar_bc, 64 * k, 0, g, it.c * Qt, it.b);
        }
    };

    PhaseCount pc_x = {0u, 0u}, pc_k = {0u, 0u}, pc_bc = {0u, 0u};
    PhaseCount pc_1 = {0u, 0u}, pc_2 = {0u, 0u}, pc_3 = {0u, 0u};
    if (tid == 0) {
        for (int i = 0; i < 6; ++i) mbar_init(&bar_x[i], 1);
        mbar_fence_init();
        tma_prefetch_desc(&tmX);
        tma_prefetch_desc(&tmDY);
        tma_prefetch_desc(&tmB);
        tma_prefetch_desc(&tmC);
        const int first = atomicAdd(chain_ticket(p), 1);   // < nitems: the grid is <= nitems
        s_item[0] = first;
        issue_x(first);
        ++pc_x.issued;
        issue_k(first);
        ++pc_k.issued;
        issue_bc(first);
        ++pc_bc.issued;
    }
    if (warp == 0) tmem_alloc(tslot, TMEM_COLS);
    if (N < NP) {   // state rows 64-127 of B / C are never loaded: keep them zero
        for (int i = tid; i < (int)(TILE / 16); i += THREADS) {
            reinterpret_cast<uint4 *>(sm + SM_B + TILE)[i] = make_uint4(0, 0, 0, 0);
            reinterpret_cast<uint4 *>(sm + SM_C + TILE)[i] = make_uint4(0, 0, 0, 0);
        }
    }
    fence_proxy_async();
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tb = *tslot;
    int item = s_item[0];
    ssdk::Tok tok;
    float alog;
    {
        const ChunkItem it = chunk_item_rcs(p, item);
        tok = ssdk::tok_load_q(p, it.b, it.h, it.c * Qt, Qt);
        alog = __ldg(p.A_log + it.h * p.ndec);
    }
    bool aborted = false;

    for (int k = 0; item < nitems; ++k) {
        if (tid == 0) s_item[1] = atomicAdd(chain_ticket(p), 1);
        const uint32_t par = (uint32_t)(k & 1);
        const ChunkItem it = chunk_item_rcs(p, item);
        const int c = it.c, h = it.h, b = it.b;
        const int g = h / p.hpg;
        const int bh = b * p.H + h, rr = p.nc - 1 - c;   // chunks of (b, h) walked before this one
        const int t0 = c * Qt;
        const long long u = bhc(p, b, h, c);
        // the previous item's stores have read their staging tiles
        if (tid == 0) bulk_wait_read_all();
        ssdk::chunk_scalars(p, f32, t0, Qt, tok, alog, f32 + F_FE);
        const int next = s_item[1];
        if (next < nitems) {
            const ChunkItem nx = chunk_item_rcs(p, next);
            tok = ssdk::tok_load_q(p, nx.b, nx.h, nx.c * Qt, Qt);
            alog = __ldg(p.A_log + nx.h * p.ndec);
            if (tid == 0) {   // the next item's tiles stream into L2 while this one runs
                const int g2 = nx.h / p.hpg;
                tma_prefetch_5d(&tmX, 0, 0, nx.h, nx.c * Qt, nx.b);
                tma_prefetch_5d(&tmDY, 0, 0, nx.h, nx.c * Qt, nx.b);
                for (int kb = 0; kb < nbox; ++kb) {
                    tma_prefetch_5d(&tmB, 64 * kb, 0, g2, nx.c * Qt, nx.b);
                    tma_prefetch_5d(&tmC, 64 * kb, 0, g2, nx.c * Qt, nx.b);
                }
                bulk_prefetch_l2(p.ws_kp + bhc(p, nx.b, nx.h, nx.c) * SLOT_FLOATS, 2 * TILE);
            }
        }
        const float a2 = f32[F_SC], E = f32[F_SC + 2];
        {
            const bool o1 = mbar_wait(bar_x, par, WAIT_LIMIT);
            const bool o2 = o1 && mbar_wait(bar_k, par, WAIT_LIMIT);
            const bool o3 = o2 && mbar_wait(bar_bc, par, WAIT_LIMIT);
            if (tid == 0) {
                pc_x.done += o1 ? 1u : 0u;
                pc_k.done += o2 ? 1u : 0u;
                pc_bc.done += o3 ? 1u : 0u;
            }
            int ok = o3 ? 1 : 0;
            if (!ok) {
                ssd_raise_error(1);
                chain_abort(p);
            }
            if (!__syncthreads_and(ok)) {
                aborted = true;
                break;
            }
        }
        // ---- phase 1a: CB = C B^T, dS = dY X^T --------------------------------------
        if (tid == 0) {
            fence_after_sync();
            const uint32_t b_base = smem_u32(sm + SM_B), c_base = smem_u32(sm + SM_C);
            const uint32_t x_base = smem_u32(sm + SM_X), dy_base = smem_u32(sm + SM_DY);
            const uint32_t id128 = idesc_bf16(128, 128, false, false);
            for (int s = 0; s < N / 16; ++s) {
                const uint32_t off = (uint32_t)(s >> 2) * TILE + (uint32_t)(s & 3) * 32u;
                mma_bf16(tb + T_CB, sdesc(c_base + off, 16u, 1024u, LAYOUT_SW128),
                         sdesc(b_base + off, 16u, 1024u, LAYOUT_SW128), id128, s > 0);
            }
            for (int s = 0; s < 4; ++s)
                mma_bf16(tb + T_DS, sdesc(dy_base + s * 32u, 16u, 1024u, LAYOUT_SW128),
                         sdesc(x_base + s * 32u, 16u, 1024u, LAYOUT_SW128), id128, s > 0);
        }
        // diag(e) dy as bf16 hi (SM_DYS) + lo (dCB's place, free until the masking), and the
        // K_in lo tile after it (same swizzled positions throughout)
        {
            const unsigned char *klo =
                reinterpret_cast<const unsigned char *>(p.ws_kp + u * SLOT_FLOATS) + TILE;
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                const int ch = tid + THREADS * q;
                const int r = ch >> 3;
                const uint32_t off = (uint32_t)r * 128u + (uint32_t)(ch & 7) * 16u;
                const float e = f32[F_EW + (r >> lgR)];
                float v[8], hi[8], lo[8];
                unpack8(*reinterpret_cast<const uint4 *>(sm + SM_DY + off), v);
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    v[j] *= e;
                    hi[j] = __bfloat162float(__float2bfloat16_rn(v[j]));
                    lo[j] = v[j] - hi[j];
                }
                *reinterpret_cast<uint4 *>(sm + SM_DYS + off) = pack8(hi);
                *reinterpret_cast<uint4 *>(sm + SM_DCB + off) = pack8(lo);
                *reinterpret_cast<uint4 *>(sm + SM_DCB + TILE + off) =
                    __ldg(reinterpret_cast<const uint4 *>(klo + off));
            }
        }
        fence_proxy_async();
        fence_before_sync();
        __syncthreads();
        // ---- phase 1b: dC <- diag(e) dY K_in^T; Y_o = C K_in (hi + lo, for R);
        //      G_loc = C^T diag(e) dY (hi + lo) ------------------------------------------
        if (tid == 0) {
            fence_after_sync();
            const uint32_t c_base = smem_u32(sm + SM_C), k_base = smem_u32(sm + SM_K);
            const uint32_t klo_base = smem_u32(sm + SM_DCB + TILE);
            const uint32_t dys_base = smem_u32(sm + SM_DYS), dyl_base = smem_u32(sm + SM_DCB);
            const uint32_t id128 = idesc_bf16(128, 128, false, false);
            // hi * hi + hi * lo + lo * hi
            const uint32_t a_of[3] = {dys_base, dys_base, dyl_base};
            const uint32_t b_of[3] = {k_base, klo_base, k_base};
            for (int part = 0; part < 3; ++part)
                for (int s = 0; s < 4; ++s)
                    mma_bf16(tb + T_DC, sdesc(a_of[part] + s * 32u, 16u, 1024u, LAYOUT_SW128),
                             sdesc(b_of[part] + s * 32u, 16u, 1024u, LAYOUT_SW128), id128,
                             part > 0 || s > 0);
            const uint32_t id_yo = idesc_bf16(128, 64, false, true);
            for (int part = 0; part < 2; ++part)
                for (int s = 0; s < N / 16; ++s)
                    mma_bf16(tb + T_YO,
                             sdesc(c_base + (uint32_t)(s >> 2) * TILE + (uint32_t)(s & 3) * 32u,
                                   16u, 1024u, LAYOUT_SW128),
                             sdesc((part ? klo_base : k_base) + s * 2048u, TILE, 1024u, LAYOUT_SW128),
                             id_yo, part > 0 || s > 0);
            const uint32_t id64 = idesc_bf16(128, 64, true, true);
            for (int part = 0; part < 2; ++part)
                for (int s = 0; s < ROWS / 16; ++s)
                    mma_bf16(tb + T_GL, sdesc(c_base + s * 2048u, TILE, 1024u, LAYOUT_SW128),
                             sdesc((part ? dyl_base : dys_base) + s * 2048u, TILE, 1024u,
                                   LAYOUT_SW128),
                             id64, part > 0 || s > 0);
            mma_commit(bar_p1);
            ++pc_1.issued;
        }
        {
            int ok = mbar_wait(bar_p1, par, WAIT_LIMIT) ? 1 : 0;
            if (tid == 0) pc_1.done += (uint32_t)ok;
            if (!ok) {
                ssd_raise_error(1);
                chain_abort(p);
            }
            fence_after_sync();
            if (ok) {
                // ---- masking: P = CB (.) W, dCB = dS (.) W, the sums of Z, and R ----------
                float cbv[32], dsv[32], colz[32];
                tmem_ld16(tb + T_CB + lane_q + 32u * cb4, *reinterpret_cast<float(*)[16]>(cbv));
                tmem_ld16(tb + T_CB + lane_q + 32u * cb4 + 16u, *reinterpret_cast<float(*)[16]>(cbv + 16));
                tmem_ld16(tb + T_DS + lane_q + 32u * cb4, *reinterpret_cast<float(*)[16]>(dsv));
                tmem_ld16(tb + T_DS + lane_q + 32u * cb4 + 16u, *reinterpret_cast<float(*)[16]>(dsv + 16));
                const int tj = row >> lgR;
                const float stj = f32[F_S + tj], gj = f32[F_GAM + tj];
                const int i0 = 32 * cb4;
                float rowz = 0.f, diag = 0.f;
#pragma unroll
                for (int q8 = 0; q8 < 4; ++q8) {
                    float pv[8], dv[8];
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const int kk = 8 * q8 + j;
                        const int ti = (i0 + kk) >> lgR;
                        const float cb = cbv[kk], ds = dsv[kk];
                        float z = 0.f, pw = 0.f, dw = 0.f;
                        if (ti < tj) {
                            const float wd = ex2_fast(a2 * (stj - f32[F_S + ti]));
                            const float sg = f32[F_SIG + ti];
                            z = ds * cb * wd;             // per unit sigma
                            rowz = fmaf(z, sg, rowz);
                            pw = cb * wd * sg;
                            dw = ds * wd * sg;
                        } else if (ti == tj) {
                            diag = fmaf(ds, cb, diag);
                            pw = cb * gj;
                            dw = ds * gj;
                        }
                        colz[kk] = z;
                        pv[j] = pw;
                        dv[j] = dw;
                    }
                    const uint32_t off = off_kmaj(row, i0 + 8 * q8, 128u, 2048u);
                    *reinterpret_cast<uint4 *>(sm + SM_P + off) = pack8(pv);
                    *reinterpret_cast<uint4 *>(sm + SM_DCB + off) = pack8(dv);
                }
                xreduce<32, 32>(colz, lane);   // lane l: column i0 + l over the warp's 32 rows
                red[R_COLZ + qd * 128 + i0 + lane] = colz[0];
                red[R_ROWZ + cb4 * 128 + row] = rowz;
                red[R_DIAG + cb4 * 128 + row] = diag;
                // R[j] = e_j <dY_j, (C K_in)_j> over this thread's 16 p
                float yo[16];
                tmem_ld16(tb + T_YO + lane_q + 16u * cb4, yo);
                float roff = 0.f;
#pragma unroll
                for (int g8 = 0; g8 < 2; ++g8) {
                    float dyv[8];
                    unpack8(*reinterpret_cast<const uint4 *>(sm + SM_DY + sw_off(row, 2 * cb4 + g8)), dyv);
#pragma unroll
                    for (int j = 0; j < 8; ++j) roff = fmaf(dyv[j], yo[8 * g8 + j], roff);
                }
                red[R_ROFF + cb4 * 128 + row] = roff * f32[F_EW + tj];
            }
            fence_proxy_async();
            fence_before_sync();
            if (!__syncthreads_and(ok)) {
                aborted = true;
                break;
            }
        }
        // ---- chain step (needs only G_loc): G_in = E G_out + G_loc; Q = <G_out, E K_in> ----
        {
            int ok = 1;
            // the adjoint leaving this chunk is published by the item of chunk c + 1
            if (tid == 0 && rr > 0 &&
                !wait_count(p.ws_flag + bh, rr, chain_abort_word(p), p.wait_limit)) {
                ssd_raise_error(2);
                chain_abort(p);
                ok = 0;
            }
            if (!__syncthreads_and(ok)) {   // also orders the wait before the loads of G_out
                aborted = true;
                break;
            }
        }
        float go[16];   // G_out of (state row `row`, 16 columns from 16 cb4), kept for phase 3
        {
            const int n = row, cq = cb4;
            float gl[16];
#pragma unroll
            for (int j4 = 0; j4 < 4; ++j4) {
                float4 a4 = make_float4(0.f, 0.f, 0.f, 0.f);
                if (rr > 0 && n < N) a4 = __ldcg(carry_ptr(p, rr & 1, bh, cq, n) + j4 * NP);
                go[4 * j4] = a4.x;
                go[4 * j4 + 1] = a4.y;
                go[4 * j4 + 2] = a4.z;
                go[4 * j4 + 3] = a4.w;
            }
            tmem_ld16(tb + T_GL + lane_q + 16u * cq, gl);
            const unsigned char *kslot =
                reinterpret_cast<const unsigned char *>(p.ws_kp + u * SLOT_FLOATS);
            float qb = 0.f;
#pragma unroll
            for (int g8 = 0; g8 < 2; ++g8) {
                const uint32_t off = sw_off(n, 2 * cq + g8);
                float kh[8], kl[8];
                unpack8(__ldg(reinterpret_cast<const uint4 *>(kslot + off)), kh);
                unpack8(__ldg(reinterpret_cast<const uint4 *>(kslot + TILE + off)), kl);
#pragma unroll
                for (int j = 0; j < 8; ++j) qb = fmaf(go[8 * g8 + j], kh[j] + kl[j], qb);
            }
            float gi[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) gi[j] = n < N ? fmaf(E, go[j], gl[j]) : 0.f;
            float db0 = 0.f;
            if (c > 0) {
                float4 *dst = carry_ptr(p, (rr + 1) & 1, bh, cq, n);
#pragma unroll
                for (int j4 = 0; j4 < 4; ++j4)
                    __stcg(dst + j4 * NP, make_float4(gi[4 * j4], gi[4 * j4 + 1], gi[4 * j4 + 2],
                                                      gi[4 * j4 + 3]));
            } else if (n < N) {
                // the adjoint of K_{-1} = h0 + beta_0 w0: dh0, dw0 = beta_0 dh0, dbeta_0
                float beta0 = 0.f;
                if (p.two_ep)
                    beta0 = (1.f - ld_io(p.lam, ix_lam(p, b, 0, h), 1)) * ld_io(p.dt, ix_dt(p, b, 0, h), 1);
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const long long i0 = ix_st(p, b, h, n, 16 * cq + j);
                    if (p.dh0) p.dh0[i0] = gi[j];
                    if (p.dw0) p.dw0[i0] = beta0 * gi[j];
                    if (p.w0) db0 = fmaf(gi[j], p.w0[i0], db0);
                }
            }
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1) {
                qb += __shfl_xor_sync(0xffffffffu, qb, o);
                db0 += __shfl_xor_sync(0xffffffffu, db0, o);
            }
            if (lane == 0) {
                f32[F_QB + warp] = qb;
                f32[F_QB + 16 + warp] = db0;
            }
        }
        fence_before_sync();
        __syncthreads();
        // the carry of chunk c - 1 is in place: let its item go (off the issue path)
        if (tid == THREADS - 32 && c > 0) publish_count(p.ws_flag + bh, rr + 1);
        // ---- phase 2: dX_d = P^T dY, dC += dCB B, dB = dCB^T C ------------------------
        if (tid == 0) {
            fence_after_sync();
            // K_in is consumed: fetch the next item's
            if (next < nitems) {
                issue_k(next);
                ++pc_k.issued;
            }
            const uint32_t p_base = smem_u32(sm + SM_P), dcb_base = smem_u32(sm + SM_DCB);
            const uint32_t b_base = smem_u32(sm + SM_B), c_base = smem_u32(sm + SM_C);
            const uint32_t dy_base = smem_u32(sm + SM_DY);
            const uint32_t id_x = idesc_bf16(128, 64, true, true);
            for (int s = 0; s < ROWS / 16; ++s)
                mma_bf16(tb + T_DXD, sdesc(p_base + s * 4096u, 2048u, 128u, LAYOUT_NONE),
                         sdesc(dy_base + s * 2048u, TILE, 1024u, LAYOUT_SW128), id_x, s > 0);
            const uint32_t id_c = idesc_bf16(128, 128, false, true);
            for (int s = 0; s < ROWS / 16; ++s)
                mma_bf16(tb + T_DC, sdesc(dcb_base + s * 256u, 128u, 2048u, LAYOUT_NONE),
                         sdesc(b_base + s * 2048u, TILE, 1024u, LAYOUT_SW128), id_c, true);
            const uint32_t id_b = idesc_bf16(128, 128, true, true);
            for (int s = 0; s < ROWS / 16; ++s)
                mma_bf16(tb + T_DB, sdesc(dcb_base + s * 4096u, 2048u, 128u, LAYOUT_NONE),
                         sdesc(c_base + s * 2048u, TILE, 1024u, LAYOUT_SW128), id_b, s > 0);
            mma_commit(bar_p2);
            ++pc_2.issued;
        }
        {
            int ok = mbar_wait(bar_p2, par, WAIT_LIMIT) ? 1 : 0;
            if (tid == 0) pc_2.done += (uint32_t)ok;
            if (!ok) {
                ssd_raise_error(1);
                chain_abort(p);
            }
            fence_after_sync();
            if (!__syncthreads_and(ok)) {
                aborted = true;
                break;
            }
        }
        // ---- phase 2 has read P and dCB: G_out hi in P's place (after 16 KB) and lo in
        // dCB's ------------------------------------------------------------------------
#pragma unroll
        for (int g8 = 0; g8 < 2; ++g8) {
            const uint32_t off = sw_off(row, 2 * cb4 + g8);
            float gh[8], glo[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                gh[j] = __bfloat162float(__float2bfloat16_rn(go[8 * g8 + j]));
                glo[j] = go[8 * g8 + j] - gh[j];
            }
            *reinterpret_cast<uint4 *>(sm + SM_P + TILE + off) = pack8(gh);
            *reinterpret_cast<uint4 *>(sm + SM_DCB + off) = pack8(glo);
        }
        fence_proxy_async();
        fence_before_sync();
        __syncthreads();
        // ---- phase 3: dX_s = B G_out, X G_out^T (G_out as hi + lo; diag(f) applied after) --
        if (tid == 0) {
            fence_after_sync();
            const uint32_t b_base = smem_u32(sm + SM_B), x_base = smem_u32(sm + SM_X);
            const uint32_t g_base = smem_u32(sm + SM_P + TILE), gl_base = smem_u32(sm + SM_DCB);
            const uint32_t id_x = idesc_bf16(128, 64, false, true);
            for (int part = 0; part < 2; ++part)
                for (int s = 0; s < N / 16; ++s)
                    mma_bf16(tb + T_DXS,
                             sdesc(b_base + (uint32_t)(s >> 2) * TILE + (uint32_t)(s & 3) * 32u,
                                   16u, 1024u, LAYOUT_SW128),
                             sdesc((part ? gl_base : g_base) + s * 2048u, TILE, 1024u, LAYOUT_SW128),
                             id_x, part > 0 || s > 0);
            const uint32_t id_b = idesc_bf16(128, 64, false, false);
            for (int nh = 0; nh < 2; ++nh)        // state rows 64 nh .. 64 nh + 63 (N = 64 each)
                for (int part = 0; part < 2; ++part)
                    for (int s = 0; s < 4; ++s)
                        mma_bf16(tb + (nh ? T_BS1 : T_BS0),
                                 sdesc(x_base + s * 32u, 16u, 1024u, LAYOUT_SW128),
                                 sdesc((part ? gl_base : g_base) + (uint32_t)nh * 8192u + s * 32u, 16u,
                                       1024u, LAYOUT_SW128),
                                 id_b, part > 0 || s > 0);
            mma_commit(bar_p3);
            ++pc_3.issued;
        }
        {
            int ok = mbar_wait(bar_p3, par, WAIT_LIMIT) ? 1 : 0;
            if (tid == 0) pc_3.done += (uint32_t)ok;
            if (!ok) {
                ssd_raise_error(1);
                chain_abort(p);
            }
            fence_after_sync();
            if (!__syncthreads_and(ok)) {
                aborted = true;
                break;
            }
        }
        // B and C are consumed: fetch the next item's
        if (tid == 0 && next < nitems) {
            issue_bc(next);
            ++pc_bc.issued;
        }
        // ---- epilogue: dx (into the e dy tile), dB (into P's place), dC (into dCB's) ----
        {
            const int ti = row >> lgR;
            const float f = f32[F_FW + ti];
            const float D = (p.R == p.O && p.D) ? __ldg(p.D + h) : 0.f;
            float dxd[16], dxs[16];
            tmem_ld16(tb + T_DXD + lane_q + 16u * cb4, dxd);
            tmem_ld16(tb + T_DXS + lane_q + 16u * cb4, dxs);
            float wq = 0.f, dd = 0.f;
#pragma unroll
            for (int g8 = 0; g8 < 2; ++g8) {
                const uint32_t off = sw_off(row, 2 * cb4 + g8);
                float xv[8], dyv[8], o8[8];
                unpack8(*reinterpret_cast<const uint4 *>(sm + SM_X + off), xv);
                unpack8(*reinterpret_cast<const uint4 *>(sm + SM_DY + off), dyv);
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const float s_ = dxs[8 * g8 + j];
                    wq = fmaf(xv[j], s_, wq);
                    dd = fmaf(dyv[j], xv[j], dd);
                    o8[j] = fmaf(D, dyv[j], fmaf(f, s_, dxd[8 * g8 + j]));
                }
                *reinterpret_cast<uint4 *>(sm + SM_DYS + off) = pack8(o8);
            }
            red[R_WQ + cb4 * 128 + row] = wq;
            red[R_DD + cb4 * 128 + row] = dd;
            const bool tvalid = t0 + ti < L;
            for (int half = 0; half < 2; ++half) {
                const uint32_t tcol = half ? T_DC : T_DB;
                float v[32];
                tmem_ld16(tb + tcol + lane_q + 32u * cb4, *reinterpret_cast<float(*)[16]>(v));
                tmem_ld16(tb + tcol + lane_q + 32u * cb4 + 16u, *reinterpret_cast<float(*)[16]>(v + 16));
                if (!half) {   // dB = (dS (.) W)^T C + diag(f) X G_out^T
                    const uint32_t ts = ((cb4 >> 1) ? T_BS1 : T_BS0) + 32u * (cb4 & 1);
                    float w2[32];
                    tmem_ld16(tb + ts + lane_q, *reinterpret_cast<float(*)[16]>(w2));
                    tmem_ld16(tb + ts + lane_q + 16u, *reinterpret_cast<float(*)[16]>(w2 + 16));
#pragma unroll
                    for (int j = 0; j < 32; ++j) v[j] = fmaf(f, w2[j], v[j]);
                }
                const int n0 = 32 * cb4;
                if (one_head) {
                    unsigned char *stg = sm + (half ? SM_DCB : SM_P) + (cb4 >> 1) * TILE;
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        float o8[8];
#pragma unroll
                        for (int j = 0; j < 8; ++j) o8[j] = v[8 * q + j];
                        *reinterpret_cast<uint4 *>(stg + sw_off(row, 4 * (cb4 & 1) + q)) = pack8(o8);
                    }
                } else if (tvalid && n0 < N && (row & Rm) < (half ? p.O : p.R)) {
                    // the (token, rank) row's own rank: a source rank of dB (< R) or a
                    // target rank of dC (< O)
                    float *dst = (half ? p.sd_dCh : p.sd_dBh) +
                                 ix_wsk(p, b, t0 + ti, h, row & Rm, half ? p.O : p.R, n0);
#pragma unroll
                    for (int q = 0; q < 8; ++q)
                        reinterpret_cast<float4 *>(dst)[q] =
                            make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
                }
            }
        }
        fence_proxy_async();
        fence_before_sync();
        __syncthreads();
        if (tid == 0) {   // rows past the sequence end are clipped by the stores
            tma_store_5d(&tmDX, sm + SM_DYS, 0, 0, h, t0, b);
            if (one_head)
                for (int kb = 0; kb < nbox; ++kb) {
                    tma_store_5d(&tmDB, sm + SM_P + kb * TILE, 64 * kb, 0, g, t0, b);
                    tma_store_5d(&tmDC, sm + SM_DCB + kb * TILE, 64 * kb, 0, g, t0, b);
                }
            bulk_commit();
        } else if (warp == 1) {
            // ---- per-token sums and the drho scans (one warp; lane: Qt / 32 tokens) --------
            const int per = Qt >> 5;
            const int R = 1 << lgR;
            float qb = 0.f, db0 = 0.f;
            for (int w = 0; w < THREADS / 32; ++w) {
                qb += f32[F_QB + w];
                db0 += f32[F_QB + 16 + w];
            }
            qb *= E;
            float cz[4], rz[4], dg[4], ro[4], wf[4], dsg[4];
            float tot_in = 0.f, tot_w = 0.f, tot_r = 0.f;
#pragma unroll
            for (int kq = 0; kq < 4; ++kq) {
                cz[kq] = rz[kq] = dg[kq] = ro[kq] = wf[kq] = dsg[kq] = 0.f;
                if (kq >= per) continue;
                const int t = lane * per + kq;
                float czs = 0.f, wq = 0.f;
                for (int j = t * R; j < t * R + R; ++j) {
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        rz[kq] += red[R_ROWZ + q * 128 + j];
                        dg[kq] += red[R_DIAG + q * 128 + j];
                        ro[kq] += red[R_ROFF + q * 128 + j];
                        czs += red[R_COLZ + q * 128 + j];
                        wq += red[R_WQ + q * 128 + j];
                    }
                }
                cz[kq] = czs * f32[F_SIG + t];
                wf[kq] = wq * f32[F_FW + t];
                dsg[kq] = czs + wq * f32[F_FE + t];
                tot_in += cz[kq] - rz[kq];
                tot_w += wf[kq];
                tot_r += ro[kq];
            }
            // exclusive prefix over lanes of (colZ - rowZ) and F; suffix of R
            float pin = tot_in, pw = tot_w, sr = tot_r;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float a_ = __shfl_up_sync(0xffffffffu, pin, o);
                const float b_ = __shfl_up_sync(0xffffffffu, pw, o);
                const float c_ = __shfl_down_sync(0xffffffffu, sr, o);
                if (lane >= o) {
                    pin += a_;
                    pw += b_;
                }
                if (lane + o < 32) sr += c_;
            }
            float run_in = pin - tot_in, run_w = pw - tot_w, run_r = sr;   // suffix includes own
            float sdr = 0.f, sdd = 0.f;
#pragma unroll
            for (int kq = 0; kq < 4; ++kq) {
                if (kq >= per) continue;
                const int t = lane * per + kq;
                const float drho = run_in + run_w + run_r + qb;
                run_in += cz[kq] - rz[kq];
                run_w += wf[kq];
                run_r -= ro[kq];
                if (t0 + t < L) {
                    float *dst = p.sd_tok + 3 * ix_bth(p, b, t0 + t, h);
                    dst[0] = dsg[kq];
                    dst[1] = dg[kq];
                    dst[2] = drho;
                    sdr = fmaf(f32[F_DT + t], drho, sdr);
                }
            }
            for (int j = lane; j < ROWS; j += 32)
                if (t0 + (j >> lgR) < L)
#pragma unroll
                    for (int q = 0; q < 4; ++q) sdd += red[R_DD + q * 128 + j];
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1) {
                sdr += __shfl_xor_sync(0xffffffffu, sdr, o);
                sdd += __shfl_xor_sync(0xffffffffu, sdd, o);
            }
            if (lane == 0) {
                p.sd_par[2 * u] = sdr;
                p.sd_par[2 * u + 1] = sdd;
                if (c == 0) p.sd_db0[bh] = db0;
            }
        }
        // x and dy are consumed: fetch the next item's
        if (tid == 0 && next < nitems) {
            issue_x(next);
            ++pc_x.issued;
        }
        fence_before_sync();
        __syncthreads();
        item = next;
    }
    if (tid == 0) bulk_wait_read_all();
    if (aborted && tid == 0) {
        drain_phases(bar_x, pc_x);
        drain_phases(bar_k, pc_k);
        drain_phases(bar_bc, pc_bc);
        drain_phases(bar_p1, pc_1);
        drain_phases(bar_p2, pc_2);
        drain_phases(bar_p3, pc_3);
    }
    fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        fence_after_sync();
        tmem_dealloc(tb, TMEM_COLS);
    }
}

// Per-token gradients of the scalar-decay backward: dgamma_t = dsigma_t +
// diag_t, dbeta_t = dsigma_{t-1} (dbeta_0 from the chain), then
//   ddt_t = lam_t dgamma_t + (1 - lam_t) dbeta_t + a drho_t,
//   dlambda_t = dt_t (dgamma_t - dbeta_t).
__global__ void k_ssd_tokens(Params p) {
    const long long total = (long long)p.Bsz * p.L * p.H;
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
         i += (long long)gridDim.x * blockDim.x) {
        const int h = (int)(i % p.H);
        const long long r = i / p.H;
        const int t = (int)(r % p.L), b = (int)(r / p.L);
        const float *tk = p.sd_tok + 3 * ix_bth(p, b, t, h);
        const float a = -expf(__ldg(p.A_log + h * p.ndec));
        const float dgam = tk[0] + tk[1];
        const float dtv = ld_io(p.dt, ix_dt(p, b, t, h), 1);
        float ddt = fmaf(a, tk[2], dgam);
        if (p.two_ep) {
            const float dbet = t > 0 ? p.sd_tok[3 * ix_bth(p, b, t - 1, h)] : p.sd_db0[b * p.H + h];
            const float lam = ld_io(p.lam, ix_lam(p, b, t, h), 1);
            ddt = fmaf(a, tk[2], fmaf(lam, dgam, (1.f - lam) * dbet));
            if (p.dlam) st_io(p.dlam, ix_lam(p, b, t, h), dtv * (dgam - dbet), 1);
        }
        st_io(p.ddt, ix_dt(p, b, t, h), ddt, 1);
    }
}

// Per-head parameter gradients: dA_log = a sum dt drho, dD = sum <dy, x>, summed over
// batch rows and chunks by one block per head in a fixed order (thread-strided
// partials, a shuffle tree per warp, then the warps in order).
constexpr int SSD_PARAM_THREADS = 256;

__global__ void __launch_bounds__(SSD_PARAM_THREADS) k_ssd_params(Params p) {
    __shared__ float s_part[2][SSD_PARAM_THREADS / 32];
    const int h = blockIdx.x, lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int n = p.Bsz * p.nc;
    float sa = 0.f, sd = 0.f;
    for (int k = threadIdx.x; k < n; k += SSD_PARAM_THREADS) {
        const int b = k / p.nc, c = k - b * p.nc;
        const long long u = chunkc::bhc(p, b, h, c);
        sa += p.sd_par[2 * u];
        sd += p.sd_par[2 * u + 1];
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) {
        sa += __shfl_xor_sync(0xffffffffu, sa, o);
        sd += __shfl_xor_sync(0xffffffffu, sd, o);
    }
    if (lane == 0) {
        s_part[0][warp] = sa;
        s_part[1][warp] = sd;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        sa = sd = 0.f;
        for (int w = 0; w < SSD_PARAM_THREADS / 32; ++w) {
            sa += s_part[0][w];
            sd += s_part[1][w];
        }
        const float a = -expf(__ldg(p.A_log + h * p.ndec));
        p.dA_log[h * p.ndec] = a * sa;
        if (p.dD) p.dD[h] = p.R == p.O ? sd : 0.f;   // D is used only when O == R
    }
}

// dB / dC of groups with several heads: the fixed-order sum of the per-head parts.
// Rank rr of a token is a source rank of dB when rr < R and a target rank of dC
// when rr < O.
__global__ void k_ssd_group_sum(Params p) {
    const int Rp = p.R > p.O ? p.R : p.O;
    const int RN = Rp * p.N;
    const long long total = (long long)p.Bsz * p.L * p.G * RN;
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
         i += (long long)gridDim.x * blockDim.x) {
        const int e = (int)(i % RN);
        const long long r = i / RN;
        const int g = (int)(r % p.G);
        const long long r2 = r / p.G;
        const int t = (int)(r2 % p.L), b = (int)(r2 / p.L);
        const int rr = e / p.N, n = e % p.N;
        // a rank past one side's count reads that side's last rank and stores nothing
        const int rb = min(rr, p.R - 1), rc = min(rr, p.O - 1);
        float sb = 0.f, sc = 0.f;
        for (int k = 0; k < p.hpg; ++k) {
            const int h = g * p.hpg + k;
            sb += p.sd_dBh[ix_wsk(p, b, t, h, rb, p.R, n)];
            sc += p.sd_dCh[ix_wsk(p, b, t, h, rc, p.O, n)];
        }
        if (rr < p.R) st_io(p.dBm, ix_B(p, b, t, g, rr, n), sb, 1);
        if (rr < p.O) st_io(p.dCm, ix_C(p, b, t, g, rr, n), sc, 1);
    }
}

namespace ssdk {

// 5-D bf16 map over (inner, rank, head-or-group, time, batch) of a tensor with R
// ranks, box (64, Rb, 1, tokens, 1) with Rb = max(R, O) >= R, 128-byte swizzle: one
// box is the chunk's 128 (token, rank) rows of 64 elements, rank rows R .. Rb - 1
// out of bounds (zero-filled by a load, dropped by a store).
static bool make_map5(CUtensorMap *m, const void *base, uint64_t inner, uint64_t R, uint32_t Rb,
                      uint64_t d2, uint64_t L, uint64_t B, uint64_t sR, uint64_t s2, uint64_t sL,
                      uint64_t sB, uint32_t Qt) {
    EncodeTiledFn fn = encode_fn();
    if (!fn || Rb < R) return false;
    cuuint64_t dims[5] = {inner, R, d2, L, B};
    cuuint64_t strides[4] = {sR * 2, s2 * 2, sL * 2, sB * 2};
    cuuint32_t box[5] = {64, Rb, 1, Qt, 1};
    cuuint32_t es[5] = {1, 1, 1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void *>(base), dims, strides, box,
              es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
           CUDA_SUCCESS;
}

}  // namespace ssdk

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
int sm_count();

static int ssd_lg_rank(int R) { return R == 1 ? 0 : (R == 2 ? 1 : (R == 4 ? 2 : -1)); }
// (token, rank) rows per token: the wider of the two ranks
static int ssd_rows_per_token(const Params &p) { return p.R > p.O ? p.R : p.O; }

// Tokens per chunk of the scalar-decay kernels (128 (token, rank) rows); R here and
// below is the rows per token, max(R, O).
// Segments of the forward: about eight work items per resident CTA, at most one
// 32 KB carry slot per CTA.
constexpr int SSD_GRID_MAX = 296;
constexpr long long SSD_ITEMS_TARGET = 8LL * SSD_GRID_MAX;
static int ssd_nchunks(long long L, int R) {
    const int qt = 128 >> (R == 4 ? 2 : R == 2 ? 1 : 0);
    return (int)((L + qt - 1) / qt);
}
static int ssd_seg_chunks(long long B, long long H, long long L, int R) {
    const long long nc = ssd_nchunks(L, R);
    long long g = (nc * B * H + SSD_ITEMS_TARGET - 1) / SSD_ITEMS_TARGET;
    if (g < 1) g = 1;
    if (g > nc) g = nc;
    return (int)g;
}
static size_t al256(size_t v) { return (v + 255) & ~size_t(255); }
// Bytes of the chain buffers: the backward's two 32 KB adjoint slots per (b, h),
// then the forward's segment states (32 KB per (segment, b, h)), segment decays and
// the per-CTA carry slots.
size_t ssd_ring_bytes(long long B, long long H, long long L, int R) {
    const size_t bh = (size_t)B * H, slot = 128 * 64 * 4;
    const int nc = ssd_nchunks(L, R), G = ssd_seg_chunks(B, H, L, R);
    const size_t nseg = (size_t)((nc + G - 1) / G);
    return al256(2 * bh * slot) + al256(nseg * bh * slot) + al256(nseg * bh * 4) +
           (size_t)SSD_GRID_MAX * slot;
}

int ssd_chunk_tokens(int R) {
    const int lg = ssd_lg_rank(R);
    return lg < 0 ? 0 : (ssdk::ROWS >> lg);
}

// Shapes the scalar-decay kernels take (alignment of the call's pointers and
// strides included).
bool ssd_supported(const Params &p) {
    auto al16 = [](const void *ptr) { return ptr == nullptr || ((uintptr_t)ptr & 15) == 0; };
    auto st16 = [](long long s) { return (s * 2) % 16 == 0; };
    return p.bf16 && !p.per_coord && p.np == 0 && p.P == 64 && (p.N == 64 || p.N == 128) &&
           ssd_lg_rank(p.R) >= 0 && ssd_lg_rank(p.O) >= 0 && p.L > 0 && al16(p.x) && al16(p.Bm) &&
           al16(p.Cm) && al16(p.y) && st16(p.sx[0]) && st16(p.sx[1]) && st16(p.sx[2]) &&
           st16(p.sy[0]) && st16(p.sy[1]) && st16(p.sy[2]) && st16(p.sB[0]) && st16(p.sB[1]) &&
           st16(p.sB[2]) && st16(p.sC[0]) && st16(p.sC[1]) && st16(p.sC[2]) &&
           chunkc::encode_fn() != nullptr;
}

template <typename K>
static cudaError_t ssd_set_smem(K kern, uint32_t bytes, bool (&done)[64]) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64 && done[dev]) return cudaSuccess;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e == cudaSuccess && dev >= 0 && dev < 64) done[dev] = true;
    return e;
}

// Forward of the scalar-decay path: y (when p.y is set), hT / last write, and
// with p.ws_kp the state entering every chunk (bf16 hi / lo tiles) for the
// backward.  Needs p.ws_ring, p.ws_flag and p.nc = chunks of ssd_chunk_tokens.
cudaError_t ssd_forward(const Params &p, cudaStream_t st) {
    using namespace ssdk;
    const int Rp = ssd_rows_per_token(p), lgR = ssd_lg_rank(Rp);
    const uint32_t Qt = (uint32_t)(ROWS >> lgR);
    CUtensorMap mx, mb, mc, my;
    if (!make_map5(&mx, p.x, 64, p.R, Rp, p.H, p.L, p.Bsz, p.P, p.sx[2], p.sx[1], p.sx[0], Qt) ||
        !make_map5(&mb, p.Bm, p.N, p.R, Rp, p.G, p.L, p.Bsz, p.N, p.sB[2], p.sB[1], p.sB[0], Qt) ||
        !make_map5(&mc, p.Cm, p.N, p.O, Rp, p.G, p.L, p.Bsz, p.N, p.sC[2], p.sC[1], p.sC[0], Qt))
        return cudaErrorInvalidValue;
    my = mx;
    if (p.y &&
        !make_map5(&my, p.y, 64, p.O, Rp, p.H, p.L, p.Bsz, p.P, p.sy[2], p.sy[1], p.sy[0], Qt))
        return cudaErrorInvalidValue;
    if (!p.ws_ring || !p.ws_flag) return cudaErrorInvalidValue;
    static bool done[64] = {}, done_s[64] = {};
    cudaError_t e;
    if ((e = ssd_set_smem(k_ssd_fwd, SMEM_BYTES, done)) != cudaSuccess) return e;
    if ((e = ssd_set_smem(k_ssd_seg_state, SMEM_BYTES, done_s)) != cudaSuccess) return e;
    if ((e = cudaMemsetAsync(p.ws_flag, 0, sizeof(int) * ((size_t)p.Bsz * p.H + 2), st)) !=
        cudaSuccess)
        return e;
    // segment buffers after the adjoint slots (see ssd_ring_bytes)
    Params q = p;
    const size_t bh = (size_t)p.Bsz * p.H, slot = 128 * 64 * 4;
    q.sd_G = ssd_seg_chunks(p.Bsz, p.H, p.L, Rp);
    q.sd_nseg = (p.nc + q.sd_G - 1) / q.sd_G;
    char *base = reinterpret_cast<char *>(p.ws_ring) + al256(2 * bh * slot);
    q.sd_seg = reinterpret_cast<float *>(base);
    base += al256((size_t)q.sd_nseg * bh * slot);
    q.sd_sege = reinterpret_cast<float *>(base);
    base += al256((size_t)q.sd_nseg * bh * 4);
    q.sd_priv = reinterpret_cast<float *>(base);
    const long long nitems = (long long)q.sd_nseg * bh;
    int cap = 2 * sm_count();
    if (cap > SSD_GRID_MAX) cap = SSD_GRID_MAX;
    const int grid = (int)(nitems < cap ? nitems : cap);
    k_ssd_seg_state<<<grid, THREADS, SMEM_BYTES, st>>>(mx, mb, q, lgR);
    profile_mark(st, "k_ssd_seg_state");
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    k_ssd_seg_pass<<<dim3(8, (unsigned)bh), 256, 0, st>>>(q);
    profile_mark(st, "k_ssd_seg_pass");
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    k_ssd_fwd<<<grid, THREADS, SMEM_BYTES, st>>>(mx, mb, mc, my, q, lgR);
    profile_mark(st, "k_ssd_fwd");
    return cudaGetLastError();
}

// Backward of the scalar-decay path.  p.ws_kp holds the state entering every
// chunk (the training forward's tiles, p.states_ready), or is filled here by a
// forward pass that writes the states only.  Needs p.ws_ring, p.ws_flag,
// p.sd_tok, p.sd_par, p.sd_db0 (and p.sd_dBh / p.sd_dCh when groups hold
// several heads).
cudaError_t ssd_backward(const Params &p, cudaStream_t st) {
    using namespace ssdk;
    cudaError_t e;
    if (!p.states_ready) {
        Params pf = p;
        pf.y = nullptr;
        pf.hT = nullptr;
        pf.wT = nullptr;
        if ((e = ssd_forward(pf, st)) != cudaSuccess) return e;
    }
    const int Rp = ssd_rows_per_token(p), lgR = ssd_lg_rank(Rp);
    const uint32_t Qt = (uint32_t)(ROWS >> lgR);
    CUtensorMap mx, mdy, mb, mc, mdx, mdb, mdc;
    if (!make_map5(&mx, p.x, 64, p.R, Rp, p.H, p.L, p.Bsz, p.P, p.sx[2], p.sx[1], p.sx[0], Qt) ||
        !make_map5(&mdy, p.dy, 64, p.O, Rp, p.H, p.L, p.Bsz, p.P, p.sy[2], p.sy[1], p.sy[0], Qt) ||
        !make_map5(&mb, p.Bm, p.N, p.R, Rp, p.G, p.L, p.Bsz, p.N, p.sB[2], p.sB[1], p.sB[0], Qt) ||
        !make_map5(&mc, p.Cm, p.N, p.O, Rp, p.G, p.L, p.Bsz, p.N, p.sC[2], p.sC[1], p.sC[0], Qt) ||
        !make_map5(&mdx, p.dx, 64, p.R, Rp, p.H, p.L, p.Bsz, p.P, p.sx[2], p.sx[1], p.sx[0], Qt))
        return cudaErrorInvalidValue;
    mdb = mb;
    mdc = mc;
    if (p.hpg == 1 &&
        (!make_map5(&mdb, p.dBm, p.N, p.R, Rp, p.G, p.L, p.Bsz, p.N, p.sB[2], p.sB[1], p.sB[0], Qt) ||
         !make_map5(&mdc, p.dCm, p.N, p.O, Rp, p.G, p.L, p.Bsz, p.N, p.sC[2], p.sC[1], p.sC[0], Qt)))
        return cudaErrorInvalidValue;
    if (!p.ws_ring || !p.ws_flag || !p.ws_kp || !p.sd_tok || !p.sd_par || !p.sd_db0 ||
        (p.hpg != 1 && (!p.sd_dBh || !p.sd_dCh)))
        return cudaErrorInvalidValue;
    static bool done[64] = {};
    if ((e = ssd_set_smem(k_ssd_bwd, ssdb::SMEM_BYTES, done)) != cudaSuccess) return e;
    if ((e = cudaMemsetAsync(p.ws_flag, 0, sizeof(int) * ((size_t)p.Bsz * p.H + 2), st)) !=
        cudaSuccess)
        return e;
    // dbeta_0 stays zero without a left endpoint
    if ((e = cudaMemsetAsync(p.sd_db0, 0, sizeof(float) * (size_t)p.Bsz * p.H, st)) != cudaSuccess)
        return e;
    const long long nitems = (long long)p.nc * p.H * p.Bsz;
    const int grid = (int)(nitems < sm_count() ? nitems : sm_count());
    k_ssd_bwd<<<grid, ssdb::THREADS, ssdb::SMEM_BYTES, st>>>(mx, mdy, mb, mc, mdx, mdb, mdc, p,
                                                             lgR);
    profile_mark(st, "k_ssd_bwd");
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const long long tot = (long long)p.Bsz * p.L * p.H;
    int blocks = (int)((tot + 255) / 256);
    if (blocks > 148 * 16) blocks = 148 * 16;
    k_ssd_tokens<<<blocks, 256, 0, st>>>(p);
    profile_mark(st, "k_ssd_tokens");
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if (p.hpg != 1) {
        const long long tg = (long long)p.Bsz * p.L * p.G * Rp * p.N;
        int gb = (int)((tg + 255) / 256);
        if (gb > 148 * 16) gb = 148 * 16;
        k_ssd_group_sum<<<gb, 256, 0, st>>>(p);
        profile_mark(st, "k_ssd_group_sum");
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    k_ssd_params<<<p.H, SSD_PARAM_THREADS, 0, st>>>(p);
    profile_mark(st, "k_ssd_params");
    return cudaGetLastError();
}

// Read and clear the device error word of these kernels.
int ssd_error_take() {
    int v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, ssm_ssd_error_word, sizeof(int)) != cudaSuccess) return -1;
    if (v) cudaMemcpyToSymbol(ssm_ssd_error_word, &zero, sizeof(int));
    return v;
}

}  // namespace ssm
