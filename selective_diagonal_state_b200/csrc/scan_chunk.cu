// Chunk-parallel tensor-core forward scan for sm_100a (bf16 I/O, fp32 state,
// SISO, head dim 64, 64 or 128 state rows).
//
// The state-mediated kernel of the scan is masked linear attention ("When a
// Diagonal State Is Not Enough", sungsoo.github.io Part 03, Thm 24): within a
// chunk, y_t = sum_{s<=t} Re(conj(c_t) Phi_{t,s} sigma_s b_s) u_s plus the
// readout of the state carried into the chunk.  With per-coordinate decays
// and 2x2 rotations the mask is not one scalar per (t, s), so the decay of
// every state mode is folded into the operands around a reference point:
//     Phi_{t,s} = exp(lam (S_t - S_ref)) exp(lam (S_ref - S_s)),  lam = a + i theta
// (the fixed-basis diagonal structure of Thm 8).  References are the starts of
// 16-token sub-blocks, so every folded factor either decays (|f| <= 1) or
// grows at most by exp(|a| * sum of 16 steps) (see k_range_check).
//
// Per chunk of Q = 64 tokens (sub-blocks i = 0..3 of 16), S_t = inclusive sum of
// dt over the chunk, Sb_i = S at the end of sub-block i-1:
//   Ci_t  = c_t conj(e^{lam (S_t - Sb_i)})           (t in block i)
//   Ch_t  = c_t conj(e^{lam S_t})                     readout of the carried state
//   Bi_s  = sigma_s b_s e^{lam (Sb_i - S_s)}          for s <= end of block i
//   Bh_s  = sigma_s b_s e^{lam (S_63 - S_s)}          chunk-end state contribution
// The two-endpoint write is used in the pre-state form
// K_t = A_t K_{t-1} + sigma_t W_t, sigma_t = gamma_t + beta_{t+1}, with
// y_t = C_t K_t - beta_{t+1} (C_t . B_t) u_t + D u_t.
//   k_chunk_fwd (persistent, chunks of a (b, h) chained through an fp32 carry)
//       scores^T_i  = Bi (64 s x N) . Ci^T (N x 16 t)          M=64,  N=16, K=N
//       Y^T         = K_c^T (64 p x N) . Ch^T (N x 64 t)       M=64,  N=64, K=N
//       S_c         = Bh^T (N x 64 s) . X (64 s x 64 p)        M=128, N=64
//       K_{c+1}     = e^{lam S_63} K_c + S_c                   elementwise, to the next chunk
//       Y^T        += X^T (64 p x s) . P^T_i (s x 16 t)        masked scores, M=64, N=16
// The backward, when it is not handed the forward's workspace, rebuilds the
// states entering every chunk with two kernels:
//   k_chunk_state_local (every chunk at once)  S_c = Bh^T X
//   k_chunk_state_pass  (chunks in order, elementwise over (row pair, p))
//                        K_c = e^{lam S_63} K_{c-1} + S_c; hT and the last write
#include <cuda.h>

#include "chunk_common.cuh"
#include "common.cuh"
#include "umma.cuh"

namespace ssm {

// Device word raised by the bounded waits of the tensor-core kernels
// (0 = no error; 1 = a wait gave up).
__device__ int ssm_chunk_error_word;
__device__ __forceinline__ void raise_error(int code) { atomicCAS(&ssm_chunk_error_word, 0, code); }

namespace chunkfwd {

using namespace umma;
using namespace chunkc;

// ============================================================================
// k_chunk_state_local: chunk-local end state S_c = Bh^T X (Bh split hi + lo, so
// the state keeps about 16 mantissa bits for the decay gradients), and the
// chunk's full decay e^{lam S_63} per mode.
// ============================================================================
namespace stl {
constexpr int THREADS = 256;
constexpr int RG = THREADS / 64;   // row groups of the operand preparation
constexpr uint32_t TMEM_COLS = 64;
constexpr uint32_t SM_B = 0;        // 16 KB raw B (two 64-row 128B-swizzled halves)
constexpr uint32_t SM_X = 16384;    // 8 KB  x (128B swizzle)
constexpr uint32_t SM_BH = 24576;   // 16 KB Bh hi, MN-major (M = state rows, K = s)
constexpr uint32_t SM_BHL = 40960;  // 16 KB Bh lo
constexpr uint32_t SM_F32 = 57344;
// the barriers follow the fp32 area, longer by the angle prefixes with per-token angles
template <bool TOK> constexpr uint32_t sm_bar() { return SM_F32 + (TOK ? F_END_TH : F_END) * 4; }
template <bool TOK> constexpr uint32_t smem_bytes() { return sm_bar<TOK>() + 64 + 1024; }
}  // namespace stl

template <bool TOK, bool ZOH>
__global__ void __launch_bounds__(stl::THREADS)
k_chunk_state_local(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmB,
                    Params p) {
    if (gated_off(p)) return;
    extern __shared__ unsigned char smem_raw[];
    unsigned char *sm = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    float *f32 = reinterpret_cast<float *>(sm + stl::SM_F32);
    uint64_t *bar_tma = reinterpret_cast<uint64_t *>(sm + stl::sm_bar<TOK>());
    uint64_t *bar_mma = bar_tma + 1;
    uint32_t *tslot = reinterpret_cast<uint32_t *>(bar_tma + 2);

    const int tid = threadIdx.x, warp = tid >> 5;
    const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int g = h / p.hpg;
    const int N = p.N, nr = p.nr, nmode = p.nr + p.np;
    const int t0 = c * Q;
    const int nbox = N / 64;

    if (tid == 0) {
        mbar_init(bar_tma, 1);
        mbar_init(bar_mma, 1);
        mbar_fence_init();
        tma_prefetch_desc(&tmX);
        tma_prefetch_desc(&tmB);
        mbar_expect_tx(bar_tma, (uint32_t)(Q * PD * 2 + Q * N * 2));
        tma_load_4d(sm + stl::SM_X, &tmX, bar_tma, 0, h, t0, b);
        for (int k = 0; k < nbox; ++k)
            tma_load_4d(sm + stl::SM_B + k * 8192, &tmB, bar_tma, 64 * k, g, t0, b);
    }
    if (warp == 0) tmem_alloc(tslot, stl::TMEM_COLS);
    mode_rates(p, f32, h);
    chunk_tokens(p, f32, b, h, t0, true);
    if constexpr (TOK) chunk_angles(p, f32, b, h, t0);
    chunk_mode_constants<TOK>(p, f32);
    for (int m = tid; m < nmode; m += stl::THREADS) {
        float *ce = p.ws_ce + bhc(p, b, h, c) * (2 * NP);
        ce[2 * m] = f32[F_KRE + fslot(0, 4) * NP + m];
        ce[2 * m + 1] = f32[F_KIM + fslot(0, 4) * NP + m];
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tacc = *tslot;
    int ok = mbar_wait(bar_tma, 0, WAIT_LIMIT) ? 1 : 0;
    if (!ok) raise_error(1);
    if (__syncthreads_and(ok)) {
        // Bh = (own-sub-block Bi) F[ib][4]; thread (t, grp) handles rows 8 (grp + RG k)
        const int t = tid & 63, grp = tid >> 6;
        const int ib = t >> 4;
        const float Sb = ib == 0 ? 0.f : f32[F_S + 16 * ib - 1];
        const float ds = f32[F_S + t] - Sb;
        // the write's scale: sigma_t, or per mode Z (ZOH, applied to b below)
        const float sig = ZOH ? 1.f : f32[F_SIG + t];
        const unsigned char *sB = sm + stl::SM_B;
        unsigned char *sv = p.sv_Bh ? p.sv_Bh + bhc(p, b, h, c) * 16384 : nullptr;
#pragma unroll 1
        for (int k = 0; k < NP / (8 * stl::RG); ++k) {
            const int r0 = 8 * (grp + stl::RG * k);
            if (r0 >= N) {
                if (!sv) break;
                // K padding of the saved tile
                *reinterpret_cast<uint4 *>(sv + off_mnmaj(r0, t, 2048u, 128u)) = make_uint4(0, 0, 0, 0);
                continue;
            }
            float rb[8], v[8];
            ld_rows8(sB, t, r0, rb);
#pragma unroll
            for (int j = 0; j < 8; j += 2) {
                const int r = r0 + j;
                if constexpr (ZOH) {
                    if (r < nr) {
                        rb[j] *= zoh_real(f32, r, t);
                        rb[j + 1] *= zoh_real(f32, r + 1, t);
                    } else {
                        const int m = nr + ((r - nr) >> 1);
                        zoh_pair<TOK>(f32, m, m - nr, t, rb[j], rb[j + 1]);
                    }
                }
                if (r < nr) {
                    v[j] = sig * rb[j] * ex2_fast(fminf(-f32[F_A2 + r] * ds, 120.f)) *
                           f32[F_KRE + fslot(ib, 4) * NP + r];
                    v[j + 1] = sig * rb[j + 1] * ex2_fast(fminf(-f32[F_A2 + r + 1] * ds, 120.f)) *
                               f32[F_KRE + fslot(ib, 4) * NP + r + 1];
                } else {
                    const int m = nr + ((r - nr) >> 1);
                    float sn, cs;
                    pair_sincos<TOK>(pair_angle<TOK>(f32, m - nr, f32[F_W + m], ds, t, 16 * ib - 1), &sn, &cs);
                    const float eb = sig * ex2_fast(fminf(-f32[F_A2 + m] * ds, 120.f));
                    const float bi0 = eb * fmaf(rb[j], cs, rb[j + 1] * sn);
                    const float bi1 = eb * fmaf(rb[j + 1], cs, -rb[j] * sn);
                    cmul(bi0, bi1, f32[F_KRE + fslot(ib, 4) * NP + m],
                         f32[F_KIM + fslot(ib, 4) * NP + m], v[j], v[j + 1]);
                }
            }
            st16_split(sm + stl::SM_BH, sm + stl::SM_BHL, off_mnmaj(r0, t, 2048u, 128u), v);
            if (sv) {  // the bf16 tile (hi part) for the backward's dx
                uint4 w;
                w.x = pack_bf16(v[0], v[1]);
                w.y = pack_bf16(v[2], v[3]);
                w.z = pack_bf16(v[4], v[5]);
                w.w = pack_bf16(v[6], v[7]);
                *reinterpret_cast<uint4 *>(sv + off_mnmaj(r0, t, 2048u, 128u)) = w;
            }
        }
        fence_proxy_async();
        fence_before_sync();
        __syncthreads();
        if (tid == 0) {
            fence_after_sync();
            const uint32_t x_base = smem_u32(sm + stl::SM_X);
            const uint32_t id = idesc_bf16(128, 64, true, true);
            for (int part = 0; part < 2; ++part) {
                const uint32_t bh_base = smem_u32(sm + (part ? stl::SM_BHL : stl::SM_BH));
                for (int s = 0; s < Q / 16; ++s)
                    mma_bf16(tacc, sdesc(bh_base + s * 4096u, 2048u, 128u, LAYOUT_NONE),
                             sdesc(x_base + s * 2048u, 8192u, 1024u, LAYOUT_SW128), id,
                             part > 0 || s > 0);
            }
            mma_commit(bar_mma);
        }
        ok = mbar_wait(bar_mma, 0, WAIT_LIMIT) ? 1 : 0;
        if (!ok) raise_error(1);
        fence_after_sync();
        if (__syncthreads_and(ok)) {
            // the chunk-local fp32 sum [N][64] at the start of the chunk's slot
            const int n = 32 * (warp & 3) + (tid & 31), half = warp >> 2;
            float *dst = p.ws_kp + bhc(p, b, h, c) * SLOT_FLOATS + n * PD;
#pragma unroll
            for (int c16 = 2 * half; c16 < 2 * half + 2; ++c16) {
                float v[16];
                tmem_ld16(tmem_addr(tacc, 32u * (warp & 3), 16u * c16), v);
                if (n < N) {
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4)
                        reinterpret_cast<float4 *>(dst + 16 * c16)[q4] =
                            make_float4(v[4 * q4], v[4 * q4 + 1], v[4 * q4 + 2], v[4 * q4 + 3]);
                }
            }
        }
    } else if (tid == 0) {
        mbar_wait(bar_tma, 0, WAIT_LIMIT);  // let an in-flight load land before exit
    }
    fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        fence_after_sync();
        tmem_dealloc(tacc, stl::TMEM_COLS);
    }
}

// ============================================================================
// k_chunk_state_pass: the carried state over the chunks of one (batch row,
// head).  Thread (row-pair group, 8 consecutive p) keeps rows 2rp, 2rp+1 for
// rp = rp0, rp0 + 32: two real modes or one rotation pair as (re, im).  Every
// chunk's loads are issued together, in 16-byte pieces.  ws_kp[c] holds S_c
// (fp32) on entry and the state entering chunk c (hi / lo tiles) on exit; the
// state after the last chunk is hT.
// ============================================================================
namespace pas {
constexpr int THREADS = 256;
constexpr int KMAX = NP / 64;   // row pairs per thread
}  // namespace pas

__global__ void __launch_bounds__(pas::THREADS) k_chunk_state_pass(Params p) {
    if (gated_off(p)) return;
    __shared__ float s_ce[3][2 * NP];   // chunk decays, triple-buffered
    const int tid = threadIdx.x;
    const int h = blockIdx.x, b = blockIdx.y;
    const int N = p.N, nr = p.nr, nc = p.nc;
    const int p8 = 8 * (tid & 7), rp0 = tid >> 3;
    const int nk = N / 64;
    // K_{-1} = h0 + beta_0 w0
    float beta0 = 0.f;
    if (p.two_ep)
        beta0 = (1.f - ld_io(p.lam, ix_lam(p, b, 0, h), 1)) * ld_io(p.dt, ix_dt(p, b, 0, h), 1);
    Rows2x8 kst[pas::KMAX];
#pragma unroll
    for (int k = 0; k < pas::KMAX; ++k) {
        const int n0 = 2 * (rp0 + 32 * k);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            float a = 0.f, d = 0.f;
            if (k < nk) {
                const long long i0 = ix_st(p, b, h, n0, p8 + j), i1 = ix_st(p, b, h, n0 + 1, p8 + j);
                if (p.h0) {
                    a = p.h0[i0];
                    d = p.h0[i1];
                }
                if (p.w0) {
                    a = fmaf(beta0, p.w0[i0], a);
                    d = fmaf(beta0, p.w0[i1], d);
                }
            }
            kst[k].a[j] = a;
            kst[k].d[j] = d;
        }
    }
    s_ce[0][tid] = __ldg(p.ws_ce + bhc(p, b, h, 0) * (2 * NP) + tid);
    // the two chunks after this one stream into L2 while this one is processed
    constexpr int PF = 2;
    for (int k = 1; k <= PF && k < nc; ++k)
        if (tid == 0) bulk_prefetch_l2(p.ws_kp + bhc(p, b, h, k) * SLOT_FLOATS, SLOT_FLOATS * 4);
    for (int c = 0; c < nc; ++c) {
        if (tid == 0 && c + PF + 1 < nc)
            bulk_prefetch_l2(p.ws_kp + bhc(p, b, h, c + PF + 1) * SLOT_FLOATS, SLOT_FLOATS * 4);
        float *slot = p.ws_kp + bhc(p, b, h, c) * SLOT_FLOATS;
        Rows2x8 sv[pas::KMAX];
#pragma unroll
        for (int k = 0; k < pas::KMAX; ++k)
            if (k < nk) rows_load_f32(slot, 2 * (rp0 + 32 * k), p8, sv[k]);
        if (c + 1 < nc) s_ce[(c + 1) % 3][tid] = __ldg(p.ws_ce + bhc(p, b, h, c + 1) * (2 * NP) + tid);
        // every thread has read its part of S_c: the slot can take the state entering chunk c
        __syncthreads();
        const float *ce = s_ce[c % 3];
        unsigned char *tile = reinterpret_cast<unsigned char *>(slot);
#pragma unroll
        for (int k = 0; k < pas::KMAX; ++k) {
            const int n0 = 2 * (rp0 + 32 * k);
            if (k >= nk) {   // rows past N read as zero by the consumers
                Rows2x8 z;
#pragma unroll
                for (int j = 0; j < 8; ++j) z.a[j] = z.d[j] = 0.f;
                rows_store_tile(tile, n0, p8, z);
                continue;
            }
            rows_store_tile(tile, n0, p8, kst[k]);
            if (n0 < nr) {
                const float e0 = ce[2 * n0], e1 = ce[2 * (n0 + 1)];
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    kst[k].a[j] = fmaf(e0, kst[k].a[j], sv[k].a[j]);
                    kst[k].d[j] = fmaf(e1, kst[k].d[j], sv[k].d[j]);
                }
            } else {
                const int m = nr + ((n0 - nr) >> 1);
                const float er = ce[2 * m], ei = ce[2 * m + 1];
#pragma unroll
                for (int j = 0; j < 8; ++j) {   // (er + i ei) (a + i d) + S
                    const float ao = kst[k].a[j], dd = kst[k].d[j];
                    kst[k].a[j] = fmaf(er, ao, fmaf(-ei, dd, sv[k].a[j]));
                    kst[k].d[j] = fmaf(er, dd, fmaf(ei, ao, sv[k].d[j]));
                }
            }
        }
    }
    // final state (beta_L = 0, so K_{L-1} = H_{L-1}) and the last write B_{L-1} u_{L-1}
    const int g = h / p.hpg, tl = p.L - 1;
#pragma unroll
    for (int k = 0; k < pas::KMAX; ++k) {
        if (k >= nk) break;
        const int n0 = 2 * (rp0 + 32 * k);
        const float b0 = p.wT ? ld_io(p.Bm, ix_B(p, b, tl, g, 0, n0), 1) : 0.f;
        const float b1 = p.wT ? ld_io(p.Bm, ix_B(p, b, tl, g, 0, n0 + 1), 1) : 0.f;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const long long i0 = ix_st(p, b, h, n0, p8 + j), i1 = ix_st(p, b, h, n0 + 1, p8 + j);
            if (p.hT) {
                p.hT[i0] = kst[k].a[j];
                p.hT[i1] = kst[k].d[j];
            }
            if (p.wT) {
                const float ul = ld_io(p.x, ix_x(p, b, tl, h, 0, p8 + j), 1);
                p.wT[i0] = b0 * ul;
                p.wT[i1] = b1 * ul;
            }
        }
    }
}

// ============================================================================
// k_chunk_fwd: the whole forward of one chunk per work item, chunks of a
// (batch row, head) chained through a carry in global memory.
//
// Items run chunk-slowest (item = c * B*H + b*H + h), one persistent CTA per SM
// taking tickets from a counter in the workspace, so the item of chunk c - 1 of
// the same (b, h) was taken B*H tickets earlier.  Per item:
//   - operands Ci, Ch, Bi (as for the scores) and Bh (hi + lo) are folded from
//     raw B / C; phase A of the tensor cores needs no carried state:
//       scores^T_i = Bi (64 s x N) . Ci^T (N x 16 t)          M=64,  N=16, K=N
//       S_c        = Bh^T (N x 64 s) . X (64 s x 64 p)        M=128, N=64 (hi, lo)
//   - K_c, the state entering the chunk, is read from a two-slot fp32 carry
//     once the item of chunk c - 1 has published it (bounded wait on a
//     per-(b, h) counter; K_0 = h0 + beta_0 w0); K_{c+1} = e^{lam S_63} K_c + S_c
//     goes to the other slot (hT and the last write after the last chunk) and
//     the counter of (b, h) is advanced.  K_c's bf16 tile feeds the readout;
//     with a saving workspace its hi / lo tiles are kept for the backward;
//   - masked scores P^T, then phase B
//       Y^T        = K_c^T (64 p x N) . Ch^T (N x 64 t)       M=64,  N=64, K=N
//                  + X^T (64 p x s) . P^T_i (s x 16 t)        M=64,  N=16
//     and y_t = Y_t + (D - beta_{t+1} C_t . B_t) u_t.
// Only the carry step sits on the chain of a (b, h), so the chain stays short
// even when B*H is below the number of SMs and the chunks of one (b, h) run
// side by side.
// The carry slots (2 x 32 KB per (b, h)) stay in L2.  Every item waits only on
// an item with a smaller ticket, which a running CTA holds, so the chain makes
// progress whatever number of CTAs is resident.
// ============================================================================
namespace fwk {
constexpr int THREADS = 512;
constexpr int RG = THREADS / 64;      // row groups of the operand preparation
constexpr uint32_t TMEM_COLS = 128;   // Y^T | scores^T (M = 64) in 0..63, S_c (M = 128) in 64..127
constexpr uint32_t SM_X = 0;          // 2 x 8 KB   x (128B swizzle, rows = t)
constexpr uint32_t SM_B = 16384;      // 16 KB raw B (two 64-row swizzled halves)
constexpr uint32_t SM_C = 32768;      // 16 KB raw C
constexpr uint32_t SM_CI = 49152;     // 16 KB Ci   K-major (64 t x 128)
constexpr uint32_t SM_CH = 65536;     // 16 KB Ch   K-major
constexpr uint32_t SM_BI = 81920;     // 40 KB Bi tiles (16, 32, 48, 64 rows)
constexpr uint32_t SM_BH = 122880;    // 16 KB Bh hi, MN-major (M = state rows, K = s)
constexpr uint32_t SM_BHL = 139264;   // 16 KB Bh lo
constexpr uint32_t SM_KT = 155648;    // 16 KB K_c hi tile (MN-major: M = 64 p, K = 128 rows)
constexpr uint32_t SM_P = 172032;     // 8 KB  P^T tiles, MN-major (N = 16 t, K = 64 s)
constexpr uint32_t SM_F32 = 180224;
// the barriers follow the fp32 area, longer by the angle prefixes with per-token angles
template <bool TOK> constexpr uint32_t sm_bar() { return SM_F32 + (TOK ? F_END_TH : F_END) * 4; }
template <bool TOK> constexpr uint32_t smem_bytes() { return sm_bar<TOK>() + 64 + 1024; }
static_assert(THREADS * 16 == 8192, "one 16-byte piece of the saved P tiles per thread");
static_assert(sm_bar<true>() % 8 == 0 && smem_bytes<true>() <= 232448, "shared memory map");
}  // namespace fwk

// K_c of thread (n, cq): the carry slot, or K_0 = h0 + beta_0 w0 for the first chunk
__device__ __forceinline__ void load_k(const Params &p, int c, int b, int h, int n, int cq,
                                       float (&kc)[16]) {
    if (n >= p.N) {
#pragma unroll
        for (int j = 0; j < 16; ++j) kc[j] = 0.f;
        return;
    }
    if (c > 0) {
        const float4 *src = carry_ptr(p, c & 1, b * p.H + h, cq, n);
#pragma unroll
        for (int j4 = 0; j4 < 4; ++j4) {
            const float4 v = __ldcg(src + j4 * NP);
            kc[4 * j4] = v.x;
            kc[4 * j4 + 1] = v.y;
            kc[4 * j4 + 2] = v.z;
            kc[4 * j4 + 3] = v.w;
        }
        return;
    }
    float beta0 = 0.f;
    if (p.two_ep)
        beta0 = (1.f - ld_io(p.lam, ix_lam(p, b, 0, h), 1)) * ld_io(p.dt, ix_dt(p, b, 0, h), 1);
#pragma unroll
    for (int j = 0; j < 16; ++j) {
        const long long i0 = ix_st(p, b, h, n, 16 * cq + j);
        float a = p.h0 ? p.h0[i0] : 0.f;
        if (p.w0) a = fmaf(beta0, p.w0[i0], a);
        kc[j] = a;
    }
}

template <bool TOK, bool ZOH>
__global__ void __launch_bounds__(fwk::THREADS, 1)
k_chunk_fwd(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmB,
            const __grid_constant__ CUtensorMap tmC, const __grid_constant__ CUtensorMap tmY,
            Params p) {
    if (gated_off(p)) return;
    const int BH = p.Bsz * p.H;
    const int nitems = p.nc * BH;
    if ((int)blockIdx.x >= nitems) return;
    extern __shared__ unsigned char smem_raw[];
    unsigned char *sm = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    float *f32 = reinterpret_cast<float *>(sm + fwk::SM_F32);
    uint64_t *bar_x = reinterpret_cast<uint64_t *>(sm + fwk::sm_bar<TOK>());   // [2] x stages
    uint64_t *bar_bc = bar_x + 2;                                       // raw B, C
    uint64_t *bar_mma = bar_x + 3;                                      // [2] phase A, B
    uint32_t *tslot = reinterpret_cast<uint32_t *>(bar_x + 5);
    int *s_item = reinterpret_cast<int *>(bar_x + 6);                  // [2] claimed tickets

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int N = p.N, nr = p.nr, L = p.L;
    const int nbox = N / 64;
    const int kn_row = 32 * (warp & 3) + lane, kcq = warp >> 2;   // carry: row, column block
    auto issue_x = [&](int item, int st) {
        const ChunkItem it = chunk_item_cs(p, item);
        mbar_expect_tx(&bar_x[st], (uint32_t)(Q * PD * 2));
        tma_load_4d(sm + fwk::SM_X + st * 8192, &tmX, &bar_x[st], 0, it.h, it.c * Q, it.b);
    };
    auto issue_bc = [&](int item) {
        const ChunkItem it = chunk_item_cs(p, item);
        const int g = it.h / p.hpg, t0 = it.c * Q;
        mbar_expect_tx(bar_bc, (uint32_t)(2 * Q * N * 2));
        for (int k = 0; k < nbox; ++k) {
            tma_load_4d(sm + fwk::SM_B + k * 8192, &tmB, bar_bc, 64 * k, g, t0, it.b);
            tma_load_4d(sm + fwk::SM_C + k * 8192, &tmC, bar_bc, 64 * k, g, t0, it.b);
        }
    };

    // phases issued / completed on each mbarrier (counted by thread 0, which issues
    // every load and the first MMA batch of a phase), for the drain of a CTA that stops
    PhaseCount pc_x[2] = {{0u, 0u}, {0u, 0u}}, pc_bc = {0u, 0u}, pc_a = {0u, 0u}, pc_b = {0u, 0u};
    if (tid == 0) {
        mbar_init(&bar_x[0], 1);
        mbar_init(&bar_x[1], 1);
        mbar_init(bar_bc, 1);
        mbar_init(&bar_mma[0], 2);   // two issuing threads commit phase A
        mbar_init(&bar_mma[1], 1);
        mbar_fence_init();
        tma_prefetch_desc(&tmX);
        tma_prefetch_desc(&tmB);
        tma_prefetch_desc(&tmC);
        const int first = atomicAdd(chain_ticket(p), 1);   // < nitems: the grid is <= nitems
        s_item[0] = first;
        issue_x(first, 0);
        ++pc_x[0].issued;
        issue_bc(first);
        ++pc_bc.issued;
    }
    if (warp == 0) tmem_alloc(tslot, fwk::TMEM_COLS);
    if (N < NP)  // K padding of Ci, Ch, Bi and M padding of Bh (rows past N are never written)
        for (int i = tid; i < (int)((fwk::SM_KT - fwk::SM_CI) / 16); i += fwk::THREADS)
            reinterpret_cast<uint4 *>(sm + fwk::SM_CI)[i] = make_uint4(0, 0, 0, 0);
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    int item = s_item[0];
    TokPrefetch tok;
    ModePrefetch mp;
    {
        const ChunkItem it = chunk_item_cs(p, item);
        tok = tok_load(p, it.b, it.h, it.c * Q);
        mp = mode_load(p, it.h);
    }
    const uint32_t tbase = *tslot;
    const uint32_t t_y = tbase;                      // Y^T (M=64, lanes 0-15 of each quarter)
    const uint32_t t_sc = tbase + (16u << 16);       // scores^T (M=64, lanes 16-31)
    const uint32_t t_s = tbase + 64u;                // S_c (M=128)
    float *cpart = reinterpret_cast<float *>(sm + fwk::SM_P);   // C.B partials until P is built
    bool aborted = false;

    for (int k = 0; item < nitems; ++k) {
        // the item after this one (read by every thread after the next barrier)
        if (tid == 0) s_item[1] = atomicAdd(chain_ticket(p), 1);
        const int st = k & 1;
        const ChunkItem it = chunk_item_cs(p, item);
        const int c = it.c, h = it.h, b = it.b;
        const int bh = b * p.H + h;
        const int t0 = c * Q;
        unsigned char *sX = sm + fwk::SM_X + st * 8192;
        const unsigned char *sB = sm + fwk::SM_B, *sC = sm + fwk::SM_C;

        // ---- this chunk's small inputs; K_c once the previous chunk has published it
        mode_rates_from(p, f32, mp);
        chunk_tokens_from(p, f32, t0, tok, true);
        if constexpr (TOK) chunk_angles(p, f32, b, h, t0);
        const int next = s_item[1];
        if (next < nitems) {
            const ChunkItem nx = chunk_item_cs(p, next);
            tok = tok_load(p, nx.b, nx.h, nx.c * Q);
            mp = mode_load(p, nx.h);
            // the other x stage was last read by the previous chunk, which is complete
            if (tid == 0) {
                issue_x(next, st ^ 1);
                ++pc_x[st ^ 1].issued;
            }
        }
        chunk_mode_constants<TOK>(p, f32);
        if (p.ws_ce && tid < p.nr + p.np) {
            float *ce = p.ws_ce + bhc(p, b, h, c) * (2 * NP);
            ce[2 * tid] = f32[F_KRE + fslot(0, 4) * NP + tid];
            ce[2 * tid + 1] = f32[F_KIM + fslot(0, 4) * NP + tid];
        }
        // the previous chunk's y store has to have read the P region (corr partials below)
        if (tid == 0) bulk_wait_read_all();
        const bool okx = mbar_wait(&bar_x[st], (uint32_t)((k >> 1) & 1), WAIT_LIMIT);
        const bool okb = okx && mbar_wait(bar_bc, (uint32_t)(k & 1), WAIT_LIMIT);
        if (tid == 0) {
            pc_x[st].done += okx ? 1u : 0u;
            pc_bc.done += okb ? 1u : 0u;
        }
        int ok = okb ? 1 : 0;
        if (!ok) {
            raise_error(1);
            chain_abort(p);
        }
        if (!__syncthreads_and(ok)) {
            aborted = true;
            break;
        }
        // ---- operand preparation: thread (t, grp) handles rows 8 (grp + RG k) ---
        {
            const int t = tid & 63, grp = tid >> 6;
            const int ib = t >> 4;
            const float Sb = ib == 0 ? 0.f : f32[F_S + 16 * ib - 1];
            const float ds = f32[F_S + t] - Sb;
            // the write's scale: sigma_t, or per mode Z (ZOH, applied to b below)
            const float sig = ZOH ? 1.f : f32[F_SIG + t];
            unsigned char *sv = p.sv_Bh ? p.sv_Bh + bhc(p, b, h, c) * 16384 : nullptr;
            float corr = 0.f;
#pragma unroll 1
            for (int kk = 0; kk < NP / (8 * fwk::RG); ++kk) {
                const int r0 = 8 * (grp + fwk::RG * kk);
                if (r0 >= N) {
                    if (!sv) break;
                    // K padding of the saved Bh tile
                    *reinterpret_cast<uint4 *>(sv + off_mnmaj(r0, t, 2048u, 128u)) = make_uint4(0, 0, 0, 0);
                    continue;
                }
                float vCI[8], vCH[8], vBI[8], vBH[8], vBX[3][8], rc[8], rb[8];
                ld_rows8(sC, t, r0, rc);
                ld_rows8(sB, t, r0, rb);
#pragma unroll
                for (int j = 0; j < 8; j += 2) {
                    const int r = r0 + j;
                    // two rows at a time: real rows r, r+1 or one pair (re, im)
                    const float c0 = rc[j], c1 = rc[j + 1];
                    float b0 = rb[j], b1 = rb[j + 1];
                    corr = fmaf(c0, b0, fmaf(c1, b1, corr));
                    if constexpr (ZOH) {
                        if (r < nr) {
                            b0 *= zoh_real(f32, r, t);
                            b1 *= zoh_real(f32, r + 1, t);
                        } else {
                            const int m = nr + ((r - nr) >> 1);
                            zoh_pair<TOK>(f32, m, m - nr, t, b0, b1);
                        }
                    }
                    if (r < nr) {
                        const int m0 = r, m1 = r + 1;
                        const float x0 = f32[F_A2 + m0] * ds, x1 = f32[F_A2 + m1] * ds;
                        const float ci0 = c0 * ex2_fast(x0), ci1 = c1 * ex2_fast(x1);
                        const float bi0 = sig * b0 * ex2_fast(fminf(-x0, 120.f));
                        const float bi1 = sig * b1 * ex2_fast(fminf(-x1, 120.f));
                        vCI[j] = ci0;
                        vCI[j + 1] = ci1;
                        vBI[j] = bi0;
                        vBI[j + 1] = bi1;
                        vBH[j] = bi0 * f32[F_KRE + fslot(ib, 4) * NP + m0];
                        vBH[j + 1] = bi1 * f32[F_KRE + fslot(ib, 4) * NP + m1];
                        const float g0 = ib ? f32[F_KRE + gslot(ib) * NP + m0] : 1.f;
                        const float g1 = ib ? f32[F_KRE + gslot(ib) * NP + m1] : 1.f;
                        vCH[j] = ci0 * g0;
                        vCH[j + 1] = ci1 * g1;
#pragma unroll
                        for (int qq = 0; qq < 3; ++qq) {
                            const int i2 = ib + 1 + qq;
                            if (i2 < 4) {
                                vBX[qq][j] = bi0 * f32[F_KRE + fslot(ib, i2) * NP + m0];
                                vBX[qq][j + 1] = bi1 * f32[F_KRE + fslot(ib, i2) * NP + m1];
                            }
                        }
                    } else {
                        const int m = nr + ((r - nr) >> 1);
                        const float x = f32[F_A2 + m] * ds;
                        float sn, cs;
                        pair_sincos<TOK>(pair_angle<TOK>(f32, m - nr, f32[F_W + m], ds, t, 16 * ib - 1), &sn,
                                         &cs);
                        // rotate by cis(-phi): (u + iv)(cs - i sn)
                        const float ec = ex2_fast(x), eb = sig * ex2_fast(fminf(-x, 120.f));
                        const float ci0 = ec * fmaf(c0, cs, c1 * sn);
                        const float ci1 = ec * fmaf(c1, cs, -c0 * sn);
                        const float bi0 = eb * fmaf(b0, cs, b1 * sn);
                        const float bi1 = eb * fmaf(b1, cs, -b0 * sn);
                        vCI[j] = ci0;
                        vCI[j + 1] = ci1;
                        vBI[j] = bi0;
                        vBI[j + 1] = bi1;
                        cmul(bi0, bi1, f32[F_KRE + fslot(ib, 4) * NP + m],
                             f32[F_KIM + fslot(ib, 4) * NP + m], vBH[j], vBH[j + 1]);
                        float gr = 1.f, gi = 0.f;
                        if (ib) {
                            gr = f32[F_KRE + gslot(ib) * NP + m];
                            gi = f32[F_KIM + gslot(ib) * NP + m];
                        }
                        cmul(ci0, ci1, gr, gi, vCH[j], vCH[j + 1]);
#pragma unroll
                        for (int qq = 0; qq < 3; ++qq) {
                            const int i2 = ib + 1 + qq;
                            if (i2 < 4)
                                cmul(bi0, bi1, f32[F_KRE + fslot(ib, i2) * NP + m],
                                     f32[F_KIM + fslot(ib, i2) * NP + m], vBX[qq][j],
                                     vBX[qq][j + 1]);
                        }
                    }
                }
                st16(sm + fwk::SM_CI, off_kmaj(t, r0, KM_LBO, KM_SBO), vCI);
                st16(sm + fwk::SM_CH, off_kmaj(t, r0, KM_LBO, KM_SBO), vCH);
                st16(sm + fwk::SM_BI + bi_off(ib), off_kmaj(t, r0, KM_LBO, KM_SBO), vBI);
#pragma unroll
                for (int qq = 0; qq < 3; ++qq) {
                    const int i2 = ib + 1 + qq;
                    if (i2 < 4)
                        st16(sm + fwk::SM_BI + bi_off(i2), off_kmaj(t, r0, KM_LBO, KM_SBO), vBX[qq]);
                }
                st16_split(sm + fwk::SM_BH, sm + fwk::SM_BHL, off_mnmaj(r0, t, 2048u, 128u), vBH);
                if (sv) {  // the bf16 Bh tile (hi part) for the backward's dx
                    uint4 w;
                    w.x = pack_bf16(vBH[0], vBH[1]);
                    w.y = pack_bf16(vBH[2], vBH[3]);
                    w.z = pack_bf16(vBH[4], vBH[5]);
                    w.w = pack_bf16(vBH[6], vBH[7]);
                    *reinterpret_cast<uint4 *>(sv + off_mnmaj(r0, t, 2048u, 128u)) = w;
                }
            }
            cpart[grp * 64 + t] = corr;
        }
        // K_c is published by the item of chunk c - 1 (everything above does not need it)
        int cw = 1;
        if (tid == 0 && c > 0 &&
            !wait_count(p.ws_flag + bh, c, chain_abort_word(p), p.wait_limit)) {
            raise_error(2);
            chain_abort(p);
            cw = 0;
        }
        fence_proxy_async();
        fence_before_sync();
        // also orders the wait before every thread's loads of K_c
        if (!__syncthreads_and(cw)) {
            aborted = true;
            break;
        }
        // raw B and C are consumed: fetch the next chunk's
        if (tid == 0 && next < nitems) {
            issue_bc(next);
            ++pc_bc.issued;
        }

        // ---- phase A: scores, chunk-local state --------------------------------
        if (tid == 0) {
            fence_after_sync();
            const uint32_t bi_base = smem_u32(sm + fwk::SM_BI), ci_base = smem_u32(sm + fwk::SM_CI);
            const uint32_t id_sc = idesc_bf16(64, 16, false, false);
            for (int i = 0; i < NSB; ++i)
                for (int s = 0; s < NP / 16; ++s)
                    mma_bf16(t_sc + 16 * i,
                             sdesc(bi_base + bi_off(i) + s * 256u, KM_LBO, KM_SBO, LAYOUT_NONE),
                             sdesc(ci_base + 2u * i * KM_SBO + s * 256u, KM_LBO, KM_SBO, LAYOUT_NONE),
                             id_sc, s > 0);
            mma_commit(&bar_mma[0]);
            ++pc_a.issued;
        } else if (tid == 32) {
            fence_after_sync();
            const uint32_t x_base = smem_u32(sX);
            const uint32_t id_s = idesc_bf16(128, 64, true, true);
            for (int part = 0; part < 2; ++part) {
                const uint32_t bh_base = smem_u32(sm + (part ? fwk::SM_BHL : fwk::SM_BH));
                for (int s = 0; s < Q / 16; ++s)
                    mma_bf16(t_s, sdesc(bh_base + s * 4096u, 2048u, 128u, LAYOUT_NONE),
                             sdesc(x_base + s * 2048u, 8192u, 1024u, LAYOUT_SW128), id_s,
                             part > 0 || s > 0);
            }
            mma_commit(&bar_mma[0]);
        }
        if (tid < 64) {
            float cs = 0.f;
#pragma unroll
            for (int kk = 0; kk < fwk::RG; ++kk) cs += cpart[kk * 64 + tid];
            const float corr = -f32[F_BN + tid] * cs + ((p.R == p.O) ? p.D[h] : 0.f);
            f32[F_CORR + tid] = corr;
            if (p.sv_corr) p.sv_corr[bhc(p, b, h, c) * Q + tid] = corr;
        }
        // K_c (fp32), in flight while the tensor cores work
        float kc[16];
        load_k(p, c, b, h, kn_row, kcq, kc);
        ok = mbar_wait(&bar_mma[0], (uint32_t)(k & 1), WAIT_LIMIT) ? 1 : 0;
        if (tid == 0) pc_a.done += (uint32_t)ok;
        if (!ok) {
            raise_error(1);
            chain_abort(p);
        }
        fence_after_sync();
        if (!__syncthreads_and(ok)) {
            aborted = true;
            break;
        }
        // K_c: bf16 tile for the readout; hi / lo tiles of the chunk's slot for the backward
        {
            unsigned char *slot = p.ws_kp
                ? reinterpret_cast<unsigned char *>(p.ws_kp + bhc(p, b, h, c) * SLOT_FLOATS)
                : nullptr;
#pragma unroll
            for (int g8 = 0; g8 < 2; ++g8) {
                const uint32_t off = off_kmaj(kn_row, 16 * kcq + 8 * g8, 128u, 1024u);
                float hi[8], lo[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const float v = kc[8 * g8 + j];
                    hi[j] = __bfloat162float(__float2bfloat16_rn(v));
                    lo[j] = v - hi[j];
                }
                st16(sm + fwk::SM_KT, off, hi);
                if (slot) {
                    st16(slot, off, hi);
                    st16(slot + TILE_BYTES, off, lo);
                }
            }
        }
        // ---- carry: K_{c+1} = e^{lam S_63} K_c + S_c (thread: row n, 16 columns) ----
        {
            float sv16[16];
            tmem_ld16(tmem_addr(t_s, 32u * (warp & 3), 16u * kcq), sv16);
            const int n = kn_row;
            const bool vrow = n < N;
            const bool pr = vrow && n >= nr;
            const bool im = pr && ((n - nr) & 1);
            const int m = pr ? nr + ((n - nr) >> 1) : (vrow ? n : 0);
            const float er = f32[F_KRE + fslot(0, 4) * NP + m];
            const float ei = pr ? f32[F_KIM + fslot(0, 4) * NP + m] : 0.f;
            float kn[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const float other = __shfl_xor_sync(0xffffffffu, kc[j], 1);
                if (!vrow)
                    kn[j] = 0.f;
                else if (!pr)
                    kn[j] = fmaf(er, kc[j], sv16[j]);
                else if (!im)   // (er + i ei)(a + i d) + S, own row = re
                    kn[j] = fmaf(er, kc[j], fmaf(-ei, other, sv16[j]));
                else            // own row = im
                    kn[j] = fmaf(er, kc[j], fmaf(ei, other, sv16[j]));
            }
            if (c + 1 < p.nc) {
                float4 *dst = carry_ptr(p, (c + 1) & 1, bh, kcq, n);
#pragma unroll
                for (int j4 = 0; j4 < 4; ++j4)
                    __stcg(dst + j4 * NP, make_float4(kn[4 * j4], kn[4 * j4 + 1], kn[4 * j4 + 2],
                                                      kn[4 * j4 + 3]));
            } else if (vrow) {
                // final state (beta_L = 0, so K_{L-1} = H_{L-1}) and the last write B_{L-1} u_{L-1}
                const int g = h / p.hpg, tl = L - 1;
                const float bl = p.wT ? ld_io(p.Bm, ix_B(p, b, tl, g, 0, n), 1) : 0.f;
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const long long i0 = ix_st(p, b, h, n, 16 * kcq + j);
                    if (p.hT) p.hT[i0] = kn[j];
                    if (p.wT) p.wT[i0] = bl * ld_io(p.x, ix_x(p, b, tl, h, 0, 16 * kcq + j), 1);
                }
            }
        }
        // ---- masked scores -> P^T tiles (two warps per TMEM lane quarter) -------
        if (warp >= 4 && warp < 12) {
            const int qd = warp & 3, i0 = 2 * ((warp - 4) >> 2);
            for (int i = i0; i < i0 + 2; ++i) {
                float v[16];
                tmem_ld16(tmem_addr(t_sc - (16u << 16), 32u * qd, 16u * i), v);
                const int sl = lane - 16;
                if (sl >= 0) {
                    const int s = 16 * qd + sl;
                    if (s < 16 * (i + 1)) {
                        float lo[8], hi[8];
#pragma unroll
                        for (int j = 0; j < 8; ++j) {
                            lo[j] = (s <= 16 * i + j) ? v[j] : 0.f;
                            hi[j] = (s <= 16 * i + 8 + j) ? v[8 + j] : 0.f;
                        }
                        unsigned char *pt = sm + fwk::SM_P + i * 2048;
                        st16(pt, off_mnmaj(0, s, 256u, 128u), lo);
                        st16(pt, off_mnmaj(8, s, 256u, 128u), hi);
                    } else if (p.sv_P) {
                        // rows past the block are zero in the saved copy (read there as P^T)
                        unsigned char *pt = sm + fwk::SM_P + i * 2048;
                        *reinterpret_cast<uint4 *>(pt + off_mnmaj(0, s, 256u, 128u)) = make_uint4(0, 0, 0, 0);
                        *reinterpret_cast<uint4 *>(pt + off_mnmaj(8, s, 256u, 128u)) = make_uint4(0, 0, 0, 0);
                    }
                }
            }
        }
        fence_proxy_async();
        fence_before_sync();
        __syncthreads();
        // the carry of (b, h) is in place: let the next chunk's item go (a thread off the
        // tensor-core issue path)
        if (tid == fwk::THREADS - 32 && c + 1 < p.nc) publish_count(p.ws_flag + bh, c + 1);
        if (p.sv_P)  // the masked score tiles, for the backward's dx (512 threads x 16 bytes)
            *reinterpret_cast<uint4 *>(p.sv_P + bhc(p, b, h, c) * 8192 + tid * 16) =
                *reinterpret_cast<const uint4 *>(sm + fwk::SM_P + tid * 16);

        // ---- phase B: Y^T = K_c^T Ch^T (readout) + X^T P^T_i (intra-chunk) ----------
        if (tid == 0) {
            fence_after_sync();
            const uint32_t kt_base = smem_u32(sm + fwk::SM_KT);
            const uint32_t ch_base = smem_u32(sm + fwk::SM_CH);
            const uint32_t id_y = idesc_bf16(64, 64, true, false);
            for (int s = 0; s < NP / 16; ++s)
                mma_bf16(t_y, sdesc(kt_base + s * 2048u, 1024u, 128u, LAYOUT_NONE),
                         sdesc(ch_base + s * 256u, KM_LBO, KM_SBO, LAYOUT_NONE), id_y, s > 0);
            const uint32_t x_base = smem_u32(sX), p_base = smem_u32(sm + fwk::SM_P);
            const uint32_t id_d = idesc_bf16(64, 16, true, true);
            for (int i = 0; i < NSB; ++i)
                for (int s = 0; s <= i; ++s)
                    mma_bf16(t_y + 16 * i, sdesc(x_base + s * 2048u, 8192u, 1024u, LAYOUT_SW128),
                             sdesc(p_base + i * 2048u + s * 512u, 256u, 128u, LAYOUT_NONE), id_d,
                             true);
            mma_commit(&bar_mma[1]);
            ++pc_b.issued;
        }
        ok = mbar_wait(&bar_mma[1], (uint32_t)(k & 1), WAIT_LIMIT) ? 1 : 0;
        if (tid == 0) pc_b.done += (uint32_t)ok;
        if (!ok) {
            raise_error(1);
            chain_abort(p);
        }
        fence_after_sync();
        if (!__syncthreads_and(ok)) {
            aborted = true;
            break;
        }
        // ---- epilogue: y_t[p] = Y^T[p][t] + corr_t u_t[p], staged in the P tiles'
        // place (phase B is done with them) and written by one TMA store --------
        {
            const int qd = warp & 3, part = warp >> 2;   // TMEM quarter, column block
            const int pp = 16 * qd + (lane & 15);
            unsigned char *ys = sm + fwk::SM_P;
            constexpr int CPW = 64 / (fwk::THREADS / 128);
            for (int c16 = 0; c16 < CPW / 16; ++c16) {
                float v[16];
                const int tc = CPW * part + 16 * c16;
                tmem_ld16(tmem_addr(t_y, 32u * qd, (uint32_t)tc), v);
                if (lane < 16) {
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const int t = tc + j;
                        const float u = bf(sX + off_sw128(t, pp));
                        *reinterpret_cast<__nv_bfloat16 *>(ys + off_sw128(t, pp)) =
                            __float2bfloat16_rn(fmaf(f32[F_CORR + t], u, v[j]));
                    }
                }
            }
        }
        fence_proxy_async();
        fence_before_sync();
        __syncthreads();
        if (tid == 0) {   // tokens past the sequence end are clipped by the store
            tma_store_4d(&tmY, sm + fwk::SM_P, 0, h, t0, b);
            bulk_commit();
        }
        item = next;
    }
    if (tid == 0) bulk_wait_read_all();
    if (aborted && tid == 0) {
        // every load and MMA still in flight lands before the CTA's shared memory and
        // TMEM go away
        drain_phases(&bar_x[0], pc_x[0]);
        drain_phases(&bar_x[1], pc_x[1]);
        drain_phases(bar_bc, pc_bc);
        drain_phases(&bar_mma[0], pc_a);
        drain_phases(&bar_mma[1], pc_b);
    }
    fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        fence_after_sync();
        tmem_dealloc(tbase, fwk::TMEM_COLS);
    }
}

}  // namespace chunkfwd

// Range condition of the folded operands.  Inside a 16-token sub-block the
// folded factors reach 2^(+-|a| log2(e) sum dt) (|a| the largest decay rate of
// the head), which must stay inside the bf16 / fp32 exponent range; a call
// where any sub-block goes past RANGE_LOG2 sets *gate, and the recurrent
// kernels take the call instead (their chain is launched behind the same gate).
constexpr float RANGE_LOG2 = 100.f;

constexpr int RANGE_HMAX = 256;   // heads whose largest rate a block tabulates once

__device__ __forceinline__ float largest_log_rate(const Params &p, int h) {
    float amax = p.A_log[h * p.ndec];
    for (int m = 1; m < p.ndec; ++m) amax = fmaxf(amax, p.A_log[h * p.ndec + m]);
    return amax;
}

__global__ void __launch_bounds__(256) k_range_check(Params p, int *gate) {
    // the largest log-rate of every head, once per block: one warp per head, its lanes
    // reading consecutive modes (fmaxf drops NaN unless every rate of the head is NaN,
    // as the sequential maximum does)
    __shared__ float s_amax[RANGE_HMAX];
    const bool tab = p.H <= RANGE_HMAX;
    if (tab) {
        const int lane = threadIdx.x & 31;
        for (int h = threadIdx.x >> 5; h < p.H; h += blockDim.x >> 5) {
            float v = __int_as_float(0x7fffffff);
            for (int m = lane; m < p.ndec; m += 32) v = fmaxf(v, p.A_log[h * p.ndec + m]);
#pragma unroll
            for (int o = 16; o; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
            if (lane == 0) s_amax[h] = v;
        }
        __syncthreads();
    }
    const int nsb = (p.L + 15) / 16;
    const long long items = (long long)p.Bsz * nsb * p.H;
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < items;
         i += (long long)gridDim.x * blockDim.x) {
        const int h = (int)(i % p.H);
        const long long r = i / p.H;
        const int sb = (int)(r % nsb), b = (int)(r / nsb);
        const float amax = tab ? s_amax[h] : largest_log_rate(p, h);
        float span = 0.f;
        for (int k = 0; k < 16; ++k) {
            const int t = 16 * sb + k;
            if (t < p.L) span += ld_io(p.dt, ix_dt(p, b, t, h), p.bf16);
        }
        if (!(expf(amax) * 1.4426950408889634f * span <= RANGE_LOG2)) *gate = 1;
    }
}

cudaError_t chunk_range_check(const Params &p, int *gate, cudaStream_t st) {
    const long long items = (long long)p.Bsz * ((p.L + 15) / 16) * p.H;
    long long blocks = (items + 255) / 256;
    if (blocks > 148 * 8) blocks = 148 * 8;
    if (blocks < 1) blocks = 1;
    k_range_check<<<(int)blocks, 256, 0, st>>>(p, gate);
    profile_mark(st, "k_range_check");
    return cudaGetLastError();
}

// Whether the tensor-core forward handles this problem.
bool chunk_fwd_supported(const Params &p) {
    auto al16 = [](const void *ptr) { return ((uintptr_t)ptr & 15) == 0; };
    auto st16 = [](long long s) { return (s * 2) % 16 == 0; };
    // y (forward) leaves by TMA stores
    const bool yok = !p.y || (al16(p.y) && st16(p.sy[0]) && st16(p.sy[1]) && st16(p.sy[2]));
    return yok && !p.nst && p.bf16 && p.P == chunkc::PD && p.R == 1 && p.O == 1 &&
           (p.N == 64 || p.N == 128) &&
           p.nr % 8 == 0 && p.L > 0 && al16(p.x) && al16(p.Bm) && al16(p.Cm) && st16(p.sx[0]) &&
           st16(p.sx[1]) && st16(p.sx[2]) && st16(p.sB[0]) && st16(p.sB[1]) && st16(p.sB[2]) &&
           st16(p.sC[0]) && st16(p.sC[1]) && st16(p.sC[2]) && chunkc::encode_fn() != nullptr;
}

// The tensor-core backward additionally reads dy through TMA, writes dx in 16-byte rows and
// dB / dC through TMA.
bool chunk_bwd_supported(const Params &p) {
    auto al16 = [](const void *ptr) { return ((uintptr_t)ptr & 15) == 0; };
    auto st16 = [](long long s) { return (s * 2) % 16 == 0; };
    // dB / dC go out by TMA stores when every group has one head
    const bool dbc = p.hpg != 1 || (al16(p.dBm) && al16(p.dCm));
    return chunk_fwd_supported(p) && p.dy && al16(p.dy) && st16(p.sy[0]) && st16(p.sy[1]) &&
           st16(p.sy[2]) && (!p.dx || al16(p.dx)) && dbc;
}

// Streaming multiprocessors of the current device (grid of the persistent kernels).
int sm_count() {
    static int cached[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    if (!cached[dev]) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1)
            n = 148;
        cached[dev] = n;
    }
    return cached[dev];
}

// Opt-in to the dynamic shared memory of a kernel on the current device (the
// attribute is per device, so the flag is kept per device ordinal).
template <typename K>
static cudaError_t set_smem_once(K kern, uint32_t bytes, bool (&done)[64]) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64 && done[dev]) return cudaSuccess;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e == cudaSuccess && dev >= 0 && dev < 64) done[dev] = true;
    return e;
}

template <bool TOK, bool ZOH>
static cudaError_t launch_state_local(const CUtensorMap &mx, const CUtensorMap &mb, const Params &p,
                                      cudaStream_t st) {
    using namespace chunkfwd;
    static bool done[64] = {};
    cudaError_t e;
    if ((e = set_smem_once(k_chunk_state_local<TOK, ZOH>, stl::smem_bytes<TOK>(), done)) !=
        cudaSuccess)
        return e;
    k_chunk_state_local<TOK, ZOH>
        <<<dim3(p.nc, p.H, p.Bsz), stl::THREADS, stl::smem_bytes<TOK>(), st>>>(mx, mb, p);
    return cudaSuccess;
}

template <bool TOK, bool ZOH>
static cudaError_t launch_fwd(const CUtensorMap &mx, const CUtensorMap &mb, const CUtensorMap &mc,
                              const CUtensorMap &my, const Params &p, int grid, cudaStream_t st) {
    using namespace chunkfwd;
    static bool done[64] = {};
    cudaError_t e;
    if ((e = set_smem_once(k_chunk_fwd<TOK, ZOH>, fwk::smem_bytes<TOK>(), done)) != cudaSuccess)
        return e;
    k_chunk_fwd<TOK, ZOH><<<grid, fwk::THREADS, fwk::smem_bytes<TOK>(), st>>>(mx, mb, mc, my, p);
    return cudaSuccess;
}

// The state entering every chunk (p.ws_kp) and the chunk decays (p.ws_ce);
// also hT and the last write when p.hT / p.wT are set.
cudaError_t chunk_states(const Params &p, cudaStream_t st) {
    using namespace chunkfwd;
    CUtensorMap mx, mb;
    if (!make_map(&mx, p.x, PD, p.H, p.L, p.Bsz, p.sx[2], p.sx[1], p.sx[0], PD, true) ||
        !make_map(&mb, p.Bm, p.N, p.G, p.L, p.Bsz, p.sB[2], p.sB[1], p.sB[0], 64, true))
        return cudaErrorInvalidValue;
    // one instantiation per angle mode and write form
    cudaError_t e = by_variant(p, [&](auto tok, auto zoh) {
        return launch_state_local<decltype(tok)::value, decltype(zoh)::value>(mx, mb, p, st);
    });
    if (e != cudaSuccess) return e;
    profile_mark(st, "k_chunk_state_local");
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    k_chunk_state_pass<<<dim3(p.H, p.Bsz), pas::THREADS, 0, st>>>(p);
    profile_mark(st, "k_chunk_state_pass");
    return cudaGetLastError();
}

cudaError_t chunk_forward(const Params &p, cudaStream_t st) {
    using namespace chunkfwd;
    CUtensorMap mx, mb, mc;
    if (!make_map(&mx, p.x, PD, p.H, p.L, p.Bsz, p.sx[2], p.sx[1], p.sx[0], PD, true) ||
        !make_map(&mb, p.Bm, p.N, p.G, p.L, p.Bsz, p.sB[2], p.sB[1], p.sB[0], 64, true) ||
        !make_map(&mc, p.Cm, p.N, p.G, p.L, p.Bsz, p.sC[2], p.sC[1], p.sC[0], 64, true))
        return cudaErrorInvalidValue;
    if (!p.ws_ring || !p.ws_flag) return cudaErrorInvalidValue;
    cudaError_t e;
    // the per-(b, h) carry counters, the ticket and the abort word start at zero on every call
    if ((e = cudaMemsetAsync(p.ws_flag, 0, sizeof(int) * ((size_t)p.Bsz * p.H + 2), st)) !=
        cudaSuccess)
        return e;
    const long long nitems = (long long)p.nc * p.H * p.Bsz;
    const int grid = (int)(nitems < sm_count() ? nitems : sm_count());
    CUtensorMap my;
    if (!make_map(&my, p.y, PD, p.H, p.L, p.Bsz, p.sy[2], p.sy[1], p.sy[0], PD, true))
        return cudaErrorInvalidValue;
    if ((e = by_variant(p, [&](auto tok, auto zoh) {
             return launch_fwd<decltype(tok)::value, decltype(zoh)::value>(mx, mb, mc, my, p, grid,
                                                                            st);
         })) != cudaSuccess)
        return e;
    profile_mark(st, "k_chunk_fwd");
    return cudaGetLastError();
}

// Read and clear the device error word of the tensor-core kernels.
int chunk_error_take() {
    int v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, ssm_chunk_error_word, sizeof(int)) != cudaSuccess) return -1;
    if (v) cudaMemcpyToSymbol(ssm_chunk_error_word, &zero, sizeof(int));
    return v;
}

}  // namespace ssm
