// Chunk-parallel reverse part of the backward scan on the tensor cores (bf16
// I/O, fp32 state, SISO, head dim 64, up to 128 state rows).
//
// The adjoint of the pre-state, Gbar_t = dL/dK_t, obeys the transposed
// recurrence Gbar_t = C_t^T dy_t + A_{t+1}^T Gbar_{t+1} ("When a Diagonal State
// Is Not Enough", sungsoo.github.io Part 01: the linear-transition recurrence,
// here run backwards).  In the complex packing of a rotation pair, A^T is the
// conjugate.  Per chunk of 64 tokens with S_t the inclusive sum of dt inside
// the chunk and Gc the adjoint carried in from later chunks (adjoint of K at
// the chunk's last token, before that token's own readout term):
//   Gbar_t = sum_{t' >= t} conj(e^{lam (S_t' - S_t)}) c_t' dy_t'  +  conj(e^{lam (S_63 - S_t)}) Gc
// so the work splits into
//   k_chunk_bwd_fused  (persistent, the chunks of every (b, h) last to first, chained
//                       through an fp32 carry in L2): the chunk-local adjoint
//                       Ghat_c = sum_t conj(e^{lam S_t}) c_t dy_t^T, the carry step
//                       Gc_{c-1} = conj(e^{lam S_63}) Gc_c + Ghat_c, and dC_t and
//                       gbu_t = sum_p u_t,p Gbar_t,p, then the decay-gradient sums of the chunk
//   k_chunk_bwd_dx     (every chunk at once)   dx_s = sum_{t>=s} P_ts dy_t + (Bh_s)^T Gc_c + corr
// where P is the masked score matrix of the forward and Bh_s = sigma_s b_s
// e^{lam (S_63 - S_s)} (the same folded operands as the chunked forward).  The
// fused kernel also forms, at every chunk start, the exact boundary value
// sum_p conj(Gc_{c-1}) K_end_{c-1} of the decay-gradient scan, and writes
// dL/dh0, dL/dw0 and dL/dbeta_0 at the first chunk.
#include <cuda.h>

#include "chunk_common.cuh"
#include "common.cuh"
#include "umma.cuh"

namespace ssm {

// Device word raised by the bounded waits of these kernels (0 = no error, 1 = a wait gave up).
__device__ int ssm_chunk_rev_error_word;
__device__ __forceinline__ void rev_raise_error(int code) {
    atomicCAS(&ssm_chunk_rev_error_word, 0, code);
}

namespace chunkrev {
using namespace umma;
using namespace chunkc;


// ============================================================================
// k_chunk_bwd_dx: per chunk,
//   DX = P^T (64 s x 64 t) . dY (64 t x 64 p)  +  Bh (64 s x N) . Gc (N x 64 p)
//   dx_s = DX_s + (D - beta_{s+1} (C_s . B_s)) dy_s
// with the scores built exactly as in the forward: scores^T_i = Bi . Ci^T.
// ============================================================================
namespace dxk {
constexpr int THREADS = 512;
constexpr int RG = THREADS / 64;   // row groups of the operand preparation
constexpr uint32_t TMEM_COLS = 64;
constexpr uint32_t SM_B = 0;          // 16 KB raw B (swizzled halves)
constexpr uint32_t SM_C = 16384;      // 16 KB raw C
constexpr uint32_t SM_DY = 32768;     // 8 KB  dy (swizzled)
constexpr uint32_t SM_CI = 40960;     // 16 KB Ci K-major (rows t, K = state rows)
constexpr uint32_t SM_BI = 57344;     // 40 KB Bi tiles (16, 32, 48, 64 rows)
constexpr uint32_t SM_BH = 98304;     // 16 KB Bh (stored MN-major with M = rows; read K-major, M = s)
constexpr uint32_t SM_P = 114688;     // 8 KB  P^T, K-major (rows s, K = t)
constexpr uint32_t SM_GC = 122880;    // 16 KB Gc bf16, MN-major B operand (N = p, K = state rows)
constexpr uint32_t SM_F32 = 139264;
// the barriers follow the fp32 area, longer by the angle prefixes with per-token angles
template <bool TOK> constexpr uint32_t sm_bar() { return SM_F32 + (TOK ? F_END_TH : F_END) * 4; }
template <bool TOK> constexpr uint32_t smem_bytes() { return sm_bar<TOK>() + 64 + 1024; }
}  // namespace dxk

template <bool TOK, bool ZOH>
__global__ void __launch_bounds__(dxk::THREADS, 1)
k_chunk_bwd_dx(const __grid_constant__ CUtensorMap tmB, const __grid_constant__ CUtensorMap tmC,
               const __grid_constant__ CUtensorMap tmDY, Params p) {
    if (gated_off(p)) return;
    extern __shared__ unsigned char smem_raw[];
    unsigned char *sm = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    float *f32 = reinterpret_cast<float *>(sm + dxk::SM_F32);
    uint64_t *bar_tma = reinterpret_cast<uint64_t *>(sm + dxk::sm_bar<TOK>());
    uint64_t *bar_mma = bar_tma + 1;   // [2]
    uint32_t *tslot = reinterpret_cast<uint32_t *>(bar_tma + 3);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int g = h / p.hpg;
    const int N = p.N, nr = p.nr, L = p.L;
    const int t0 = c * Q;
    const int nbox = N / 64;

    if (tid == 0) {
        mbar_init(bar_tma, 1);
        mbar_init(&bar_mma[0], 1);
        mbar_init(&bar_mma[1], 1);
        mbar_fence_init();
        tma_prefetch_desc(&tmB);
        tma_prefetch_desc(&tmC);
        tma_prefetch_desc(&tmDY);
        mbar_expect_tx(bar_tma, (uint32_t)(Q * PD * 2 + 2 * Q * N * 2) + TILE_BYTES);
        tma_load_4d(sm + dxk::SM_DY, &tmDY, bar_tma, 0, h, t0, b);
        // the adjoint carried into this chunk (bf16 tile: B operand, N = p, K = rows)
        bulk_load(sm + dxk::SM_GC, p.ws_gc + bhc(p, b, h, c) * SLOT_FLOATS, TILE_BYTES, bar_tma);
        for (int k = 0; k < nbox; ++k) {
            tma_load_4d(sm + dxk::SM_B + k * 8192, &tmB, bar_tma, 64 * k, g, t0, b);
            tma_load_4d(sm + dxk::SM_C + k * 8192, &tmC, bar_tma, 64 * k, g, t0, b);
        }
    }
    if (warp == 0) tmem_alloc(tslot, dxk::TMEM_COLS);
    mode_rates(p, f32, h);
    if (N < NP)  // K padding of Ci, Bi, Bh
        for (int i = tid; i < (int)((dxk::SM_P - dxk::SM_CI) / 16); i += dxk::THREADS)
            reinterpret_cast<uint4 *>(sm + dxk::SM_CI)[i] = make_uint4(0, 0, 0, 0);
    chunk_tokens(p, f32, b, h, t0, true);
    if constexpr (TOK) chunk_angles(p, f32, b, h, t0);
    chunk_mode_constants<TOK>(p, f32);
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tbase = *tslot;
    const uint32_t t_dx = tbase;                  // DX (M=64: lanes 0-15 of each quarter), cols 0..63
    const uint32_t t_sc = tbase + (16u << 16);    // scores^T (M=64: lanes 16-31), cols 0..63
    int ok = mbar_wait(bar_tma, 0, WAIT_LIMIT) ? 1 : 0;
    if (!ok) rev_raise_error(1);
    if (__syncthreads_and(ok)) {
        // ---- operands: Ci, Bi (own block and later blocks), Bh; C.B partials
        {
            const int t = tid & 63, grp = tid >> 6;
            const int ib = t >> 4;
            const float Sb = ib == 0 ? 0.f : f32[F_S + 16 * ib - 1];
            const float ds = f32[F_S + t] - Sb;
            // the write's scale: sigma_t, or per mode Z (ZOH, applied to b below)
            const float sig = ZOH ? 1.f : f32[F_SIG + t];
            const unsigned char *sB = sm + dxk::SM_B, *sC = sm + dxk::SM_C;
            float corr = 0.f;
#pragma unroll 1
            for (int k = 0; k < NP / (8 * dxk::RG); ++k) {
                const int r0 = 8 * (grp + dxk::RG * k);
                if (r0 >= N) break;
                float vCI[8], vBI[8], vBH[8], vBX[3][8], rc[8], rb[8];
                ld_rows8(sC, t, r0, rc);
                ld_rows8(sB, t, r0, rb);
#pragma unroll
                for (int j = 0; j < 8; j += 2) {
                    const int r = r0 + j;
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
                        vCI[j] = c0 * ex2_fast(x0);
                        vCI[j + 1] = c1 * ex2_fast(x1);
                        const float bi0 = sig * b0 * ex2_fast(fminf(-x0, 120.f));
                        const float bi1 = sig * b1 * ex2_fast(fminf(-x1, 120.f));
                        vBI[j] = bi0;
                        vBI[j + 1] = bi1;
                        vBH[j] = bi0 * f32[F_KRE + fslot(ib, 4) * NP + m0];
                        vBH[j + 1] = bi1 * f32[F_KRE + fslot(ib, 4) * NP + m1];
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
                        pair_sincos<TOK>(pair_angle<TOK>(f32, m - nr, f32[F_W + m], ds, t, 16 * ib - 1),
                                         &sn, &cs);
                        const float ec = ex2_fast(x), eb = sig * ex2_fast(fminf(-x, 120.f));
                        vCI[j] = ec * fmaf(c0, cs, c1 * sn);
                        vCI[j + 1] = ec * fmaf(c1, cs, -c0 * sn);
                        const float bi0 = eb * fmaf(b0, cs, b1 * sn);
                        const float bi1 = eb * fmaf(b1, cs, -b0 * sn);
                        vBI[j] = bi0;
                        vBI[j + 1] = bi1;
                        cmul(bi0, bi1, f32[F_KRE + fslot(ib, 4) * NP + m],
                             f32[F_KIM + fslot(ib, 4) * NP + m], vBH[j], vBH[j + 1]);
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
                st16(sm + dxk::SM_CI, off_kmaj(t, r0, KM_LBO, KM_SBO), vCI);
                st16(sm + dxk::SM_BI + bi_off(ib), off_kmaj(t, r0, KM_LBO, KM_SBO), vBI);
#pragma unroll
                for (int qq = 0; qq < 3; ++qq) {
                    const int i2 = ib + 1 + qq;
                    if (i2 < 4)
                        st16(sm + dxk::SM_BI + bi_off(i2), off_kmaj(t, r0, KM_LBO, KM_SBO), vBX[qq]);
                }
                st16(sm + dxk::SM_BH, off_mnmaj(r0, t, 2048u, 128u), vBH);
            }
            reinterpret_cast<float *>(sm + dxk::SM_P)[grp * 64 + t] = corr;   // P is written later
        }
        fence_proxy_async();
        fence_before_sync();
        __syncthreads();

        // ---- phase A: scores^T_i = Bi . Ci^T ; DX = Bh . Gc
        if (tid == 0) {
            fence_after_sync();
            const uint32_t bi_base = smem_u32(sm + dxk::SM_BI), ci_base = smem_u32(sm + dxk::SM_CI);
            const uint32_t id_sc = idesc_bf16(64, 16, false, false);
            for (int i = 0; i < NSB; ++i)
                for (int s = 0; s < NP / 16; ++s)
                    mma_bf16(t_sc + 16 * i,
                             sdesc(bi_base + bi_off(i) + s * 256u, KM_LBO, KM_SBO, LAYOUT_NONE),
                             sdesc(ci_base + 2u * i * KM_SBO + s * 256u, KM_LBO, KM_SBO, LAYOUT_NONE),
                             id_sc, s > 0);
            const uint32_t bh_base = smem_u32(sm + dxk::SM_BH), gc_base = smem_u32(sm + dxk::SM_GC);
            const uint32_t id_dx = idesc_bf16(64, 64, false, true);
            for (int s = 0; s < NP / 16; ++s)
                mma_bf16(t_dx, sdesc(bh_base + s * 256u, 128u, 2048u, LAYOUT_NONE),
                         sdesc(gc_base + s * 2048u, 1024u, 128u, LAYOUT_NONE), id_dx, s > 0);
            mma_commit(&bar_mma[0]);
        }
        if (tid < 64) {
            float cs = 0.f;
#pragma unroll
            for (int k = 0; k < dxk::RG; ++k) cs += reinterpret_cast<const float *>(sm + dxk::SM_P)[k * 64 + tid];
            f32[F_CORR + tid] = -f32[F_BN + tid] * cs + ((p.R == p.O) ? p.D[h] : 0.f);
        }
        ok = mbar_wait(&bar_mma[0], 0, WAIT_LIMIT) ? 1 : 0;
        if (!ok) rev_raise_error(1);
        fence_after_sync();
        if (__syncthreads_and(ok)) {
            // ---- masked scores -> P^T (K-major rows s, K = t), zero where s > t
            if (warp >= 4 && warp < 12) {   // two warps per TMEM lane quarter, two blocks each
                const int qd = warp & 3, i0 = 2 * ((warp - 4) >> 2);
                for (int i = i0; i < i0 + 2; ++i) {
                    float v[16];
                    tmem_ld16(tmem_addr(t_sc - (16u << 16), 32u * qd, 16u * i), v);
                    const int sl = lane - 16;
                    if (sl >= 0) {
                        const int s = 16 * qd + sl;
                        float lo[8], hi[8];
#pragma unroll
                        for (int j = 0; j < 8; ++j) {
                            lo[j] = (s <= 16 * i + j) ? v[j] : 0.f;
                            hi[j] = (s <= 16 * i + 8 + j) ? v[8 + j] : 0.f;
                        }
                        st16(sm + dxk::SM_P, off_kmaj(s, 16 * i, 128u, 1024u), lo);
                        st16(sm + dxk::SM_P, off_kmaj(s, 16 * i + 8, 128u, 1024u), hi);
                    }
                }
            }
            fence_proxy_async();
            fence_before_sync();
            __syncthreads();
            // ---- phase B: DX += P^T dY
            if (tid == 0) {
                fence_after_sync();
                const uint32_t p_base = smem_u32(sm + dxk::SM_P), dy_base = smem_u32(sm + dxk::SM_DY);
                const uint32_t id_d = idesc_bf16(64, 64, false, true);
                for (int s = 0; s < Q / 16; ++s)
                    mma_bf16(t_dx, sdesc(p_base + s * 256u, 128u, 1024u, LAYOUT_NONE),
                             sdesc(dy_base + s * 2048u, 8192u, 1024u, LAYOUT_SW128), id_d, true);
                mma_commit(&bar_mma[1]);
            }
            ok = mbar_wait(&bar_mma[1], 0, WAIT_LIMIT) ? 1 : 0;
            if (!ok) rev_raise_error(1);
            fence_after_sync();
            if (__syncthreads_and(ok)) {
                // ---- epilogue: dx_s = DX_s + corr_s dy_s
                const int qd = warp & 3, half = warp >> 2;   // columns split over THREADS / 128 warp sets
                constexpr int CPW = 64 / (dxk::THREADS / 128);
                const int s = 16 * qd + (lane & 15);
                const unsigned char *sDY = sm + dxk::SM_DY;
                __nv_bfloat16 *xrow = reinterpret_cast<__nv_bfloat16 *>(p.dx) + b * p.sx[0] +
                                      (long long)(t0 + s) * p.sx[1] + h * p.sx[2];
                const float cr = f32[F_CORR + s];
                for (int c16 = 0; c16 < CPW / 16; ++c16) {
                    float v[16];
                    const int pc = CPW * half + 16 * c16;
                    tmem_ld16(tmem_addr(t_dx, 32u * qd, (uint32_t)pc), v);
                    if (lane < 16 && t0 + s < L) {
#pragma unroll
                        for (int hh = 0; hh < 2; ++hh) {
                            float o[8];
#pragma unroll
                            for (int j = 0; j < 8; ++j)
                                o[j] = fmaf(cr, bf(sDY + off_sw128(s, pc + 8 * hh + j)), v[8 * hh + j]);
                            uint4 w;
                            w.x = pack_bf16(o[0], o[1]);
                            w.y = pack_bf16(o[2], o[3]);
                            w.z = pack_bf16(o[4], o[5]);
                            w.w = pack_bf16(o[6], o[7]);
                            *reinterpret_cast<uint4 *>(xrow + pc + 8 * hh) = w;
                        }
                    }
                }
            }
        }
    } else if (tid == 0) {
        mbar_wait(bar_tma, 0, WAIT_LIMIT);
    }
    fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        fence_after_sync();
        tmem_dealloc(tbase, dxk::TMEM_COLS);
    }
}

// ============================================================================
// k_chunk_bwd_dx_saved: dx from the per-chunk products the training forward
// saved (masked score tiles P^T, the chunk-end folded B, the diagonal
// correction), so no operand has to be rebuilt:
//   DX = P^T (64 s x 64 t) . dY (64 t x 64 p) + Bh (64 s x N) . Gc (N x 64 p)
//   dx_s = DX_s + (D - beta_{s+1} C_s . B_s) dy_s
// Small shared memory: several CTAs share an SM.
// ============================================================================
namespace dxs {
constexpr int THREADS = 256;
constexpr uint32_t TMEM_COLS = 64;
constexpr uint32_t SM_DY = 0;        // 8 KB  dy (128B swizzle)
constexpr uint32_t SM_P = 8192;      // 8 KB  P^T, four 16-token tiles (K-major rows s)
constexpr uint32_t SM_BH = 16384;    // 16 KB Bh (stored MN-major with M = rows; read K-major, M = s)
constexpr uint32_t SM_GC = 32768;    // 16 KB Gc bf16, MN-major B operand (N = p, K = rows)
constexpr uint32_t SM_CORR = 49152;  // 64 floats
constexpr uint32_t SM_BAR = SM_CORR + 256;
constexpr uint32_t SMEM_BYTES = SM_BAR + 64 + 1024;
}  // namespace dxs

__global__ void __launch_bounds__(dxs::THREADS)
k_chunk_bwd_dx_saved(const __grid_constant__ CUtensorMap tmDY, Params p) {
    if (gated_off(p)) return;
    extern __shared__ unsigned char smem_raw[];
    unsigned char *sm = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    float *corr = reinterpret_cast<float *>(sm + dxs::SM_CORR);
    uint64_t *bar_tma = reinterpret_cast<uint64_t *>(sm + dxs::SM_BAR);
    uint64_t *bar_mma = bar_tma + 1;
    uint32_t *tslot = reinterpret_cast<uint32_t *>(bar_tma + 2);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int L = p.L;
    const int t0 = c * Q;
    const long long u = bhc(p, b, h, c);

    if (tid == 0) {
        mbar_init(bar_tma, 1);
        mbar_init(bar_mma, 1);
        mbar_fence_init();
        tma_prefetch_desc(&tmDY);
        mbar_expect_tx(bar_tma, 8192u + 8192u + 16384u + TILE_BYTES);
        tma_load_4d(sm + dxs::SM_DY, &tmDY, bar_tma, 0, h, t0, b);
        bulk_load(sm + dxs::SM_GC, p.ws_gc + u * SLOT_FLOATS, TILE_BYTES, bar_tma);
        bulk_load(sm + dxs::SM_P, p.sv_P + u * 8192, 8192u, bar_tma);
        bulk_load(sm + dxs::SM_BH, p.sv_Bh + u * 16384, 16384u, bar_tma);
    }
    if (warp == 0) tmem_alloc(tslot, dxs::TMEM_COLS);
    if (tid < Q) corr[tid] = p.sv_corr[u * Q + tid];
    fence_proxy_async();
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t t_dx = *tslot;
    int ok = mbar_wait(bar_tma, 0, WAIT_LIMIT) ? 1 : 0;
    if (!ok) rev_raise_error(1);
    if (__syncthreads_and(ok)) {
        if (tid == 0) {
            fence_after_sync();
            const uint32_t id = idesc_bf16(64, 64, false, true);
            const uint32_t p_base = smem_u32(sm + dxs::SM_P), dy_base = smem_u32(sm + dxs::SM_DY);
            for (int i = 0; i < NSB; ++i)
                mma_bf16(t_dx, sdesc(p_base + i * 2048u, 128u, 256u, LAYOUT_NONE),
                         sdesc(dy_base + i * 2048u, 8192u, 1024u, LAYOUT_SW128), id, i > 0);
            const uint32_t bh_base = smem_u32(sm + dxs::SM_BH), gc_base = smem_u32(sm + dxs::SM_GC);
            for (int s = 0; s < NP / 16; ++s)
                mma_bf16(t_dx, sdesc(bh_base + s * 256u, 128u, 2048u, LAYOUT_NONE),
                         sdesc(gc_base + s * 2048u, 1024u, 128u, LAYOUT_NONE), id, true);
            mma_commit(bar_mma);
        }
        ok = mbar_wait(bar_mma, 0, WAIT_LIMIT) ? 1 : 0;
        if (!ok) rev_raise_error(1);
        fence_after_sync();
        if (__syncthreads_and(ok)) {
            // dx_s = DX_s + corr_s dy_s; warp (quarter qd, half) takes 32 columns of 16 rows
            const int qd = warp & 3, half = warp >> 2;
            const int s = 16 * qd + (lane & 15);
            const unsigned char *sDY = sm + dxs::SM_DY;
            __nv_bfloat16 *xrow = reinterpret_cast<__nv_bfloat16 *>(p.dx) + b * p.sx[0] +
                                  (long long)(t0 + s) * p.sx[1] + h * p.sx[2];
            const float cr = corr[s];
#pragma unroll
            for (int c16 = 0; c16 < 2; ++c16) {
                float v[16];
                const int pc = 32 * half + 16 * c16;
                tmem_ld16(tmem_addr(t_dx, 32u * qd, (uint32_t)pc), v);
                if (lane < 16 && t0 + s < L) {
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        float o[8];
#pragma unroll
                        for (int j = 0; j < 8; ++j)
                            o[j] = fmaf(cr, bf(sDY + off_sw128(s, pc + 8 * hh + j)), v[8 * hh + j]);
                        uint4 w;
                        w.x = pack_bf16(o[0], o[1]);
                        w.y = pack_bf16(o[2], o[3]);
                        w.z = pack_bf16(o[4], o[5]);
                        w.w = pack_bf16(o[6], o[7]);
                        *reinterpret_cast<uint4 *>(xrow + pc + 8 * hh) = w;
                    }
                }
            }
        }
    } else if (tid == 0) {
        mbar_wait(bar_tma, 0, WAIT_LIMIT);
    }
    fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        fence_after_sync();
        tmem_dealloc(t_dx, dxs::TMEM_COLS);
    }
}

// ============================================================================
// k_chunk_bwd_fused: per chunk, the per-token backward quantities that need
// both directions inside the chunk.
//
// Forward direction (dC): with K_prev the state entering the chunk and Bo_s =
// sigma_s b_s e^{lam (Sb_k - S_s)} folded at its own sub-block's start, for t
// in sub-block i
//   dCK_t = e^{lam S_t} (dy_t . K_prev)
//         + e^{lam (S_t - Sb_i)} sum_{k <= i} F[k][i] sum_{s in block k, s <= t} (dy_t . u_s) Bo_s
// and dC_t = dCK_t - beta_{t+1} (dy_t . u_t) B_t.
// Reverse direction (gbu = sum_p u_t,p Gbar_t,p): with Gc the adjoint carried
// into the chunk and Cm_t' = conj(e^{lam (S_t' - Se_k)}) c_t' folded at its own
// sub-block's end, for t in sub-block j
//   gbu_t = conj(e^{lam (Se_j - S_t)}) [ conj(F[j+1][4]) (Gc u_t)
//           + sum_{k >= j} conj(F[j+1][k+1]) sum_{t' in block k, t' >= t} (u_t . dy_t') Cm_t' ]
// The per-row factors F are applied to accumulators after the contractions
// over tokens.  Tensor cores (operands split into bf16 hi + lo where rounding
// reaches the decay gradients):
//   V       = K_prev (N x 64 p) . dY^T (64 p x 64 t)               M=128, N=64
//   V2      = Gc (N x 64 p) . X^T (64 p x 64 t)                    M=128, N=64
//   G       = dY (64 t x 64 p) . X^T (64 p x 64 s)  [masked s <= t] M=64,  N=64
//   D_{i,k} = Bo_k^T (N x 16 s) . G_{i,k}^T (16 s x 16 t)          M=128, N=16 (k <= i)
//   E_{j,k} = Cm_k (N x 16 t') . G_{k,j} (16 t' x 16 t)             M=128, N=16 (k >= j)
// where one stored copy of the masked G serves both: K-major for D, read
// MN-major (its transpose) for E.  The epilogue then forms, per state mode,
// the within-chunk suffix sums of the decay-gradient identity (X_t - Y_t,
// X = conj(c) dCK, Y = b conj(sigma gbu)), the local part of ddt, the chunk's
// totals, dsigma_t, <dy_t, u_t>, and dB / dC (one head per group) or the
// per-head dC and gbu (several heads per group).
// ============================================================================
namespace fuk {
constexpr int THREADS = 512;
constexpr int RG = THREADS / 64;    // row groups of the operand preparation
constexpr int TQ = THREADS / 128;   // token groups of the unfold (one sub-block each)
constexpr int TPT = Q / TQ;
static_assert(TPT == 16, "the unfold takes one 16-token sub-block per thread");
constexpr uint32_t TMEM_COLS = 512;   // V 0 | V2 64 | G 128 | D_{i,k} 192.. | E_{j,k} 352..
constexpr uint32_t SM_X = 0;          // 8 KB  x (128B swizzle)
constexpr uint32_t SM_DY = 8192;      // 8 KB  dy (128B swizzle)
constexpr uint32_t SM_B = 16384;      // 16 KB raw B (two 64-row swizzled halves)
constexpr uint32_t SM_C = 32768;      // 16 KB raw C
constexpr uint32_t SM_BO = 49152;     // 16 KB Bo hi (rows s, K = state rows)
constexpr uint32_t SM_BOL = 65536;    // 16 KB Bo lo
constexpr uint32_t SM_CM = 81920;     // 16 KB Cm hi (same layout)
constexpr uint32_t SM_CML = 98304;    // 16 KB Cm lo
constexpr uint32_t SM_GM = 114688;    // 8 KB  masked G hi: 4 tiles of 16 rows t, K = s
constexpr uint32_t SM_GML = 122880;   // 8 KB  masked G lo
constexpr uint32_t SM_KT = 131072;    // 16 KB K_prev hi (rows n, K = p)
constexpr uint32_t SM_KTL = 147456;   // 16 KB K_prev lo
constexpr uint32_t SM_GC = 163840;    // 16 KB Gc hi (rows n, K = p)
constexpr uint32_t SM_GCL = 180224;   // 16 KB Gc lo
constexpr uint32_t SM_F32 = 196608;
// the barriers follow the fp32 area, longer by the angle prefixes with per-token angles
template <bool TOK> constexpr uint32_t sm_bar() { return SM_F32 + (TOK ? F_END_TH : F_END) * 4; }
template <bool TOK> constexpr uint32_t smem_bytes() { return sm_bar<TOK>() + 64 + 1024; }
static_assert(smem_bytes<true>() <= 232448, "shared memory map");
constexpr int RED_LD = 65;            // row stride of the column reductions (floats)
// after phase B the Bo .. G regions are free: two [128][RED_LD] reductions and exchange space
constexpr uint32_t SM_RED = SM_BO;
constexpr uint32_t SM_RED2 = SM_RED + 128 * RED_LD * 4;
constexpr uint32_t SM_XCH = SM_RED2 + 128 * RED_LD * 4;
static_assert(SM_XCH + 8192 <= SM_KT, "reduction space");
}  // namespace fuk

__device__ __forceinline__ uint32_t d_col(int i, int k) {   // k <= i
    return 192u + 16u * (uint32_t)(i * (i + 1) / 2 + k);
}
__device__ __forceinline__ uint32_t e_col(int j, int k) {   // k >= j
    return 352u + 16u * (uint32_t)((j == 0 ? 0 : (j == 1 ? 4 : (j == 2 ? 7 : 9))) + (k - j));
}

template <bool TOK, bool ZOH>
__global__ void __launch_bounds__(fuk::THREADS, 1)
k_chunk_bwd_fused(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmB,
                  const __grid_constant__ CUtensorMap tmC, const __grid_constant__ CUtensorMap tmDY,
                  const __grid_constant__ CUtensorMap tmDB, const __grid_constant__ CUtensorMap tmDC,
                  Params p) {
    if (gated_off(p)) return;
    const int nitems = p.nc * p.H * p.Bsz;
    if ((int)blockIdx.x >= nitems) return;
    extern __shared__ unsigned char smem_raw[];
    unsigned char *sm = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    float *f32 = reinterpret_cast<float *>(sm + fuk::SM_F32);
    uint64_t *bar_in = reinterpret_cast<uint64_t *>(sm + fuk::sm_bar<TOK>());   // [2]: x/dy/states, B/C
    uint64_t *bar_mma = bar_in + 2;                                      // [3] phases A, B, C
    uint32_t *tslot = reinterpret_cast<uint32_t *>(bar_in + 5);
    int *s_item = reinterpret_cast<int *>(bar_in + 6);                  // [2] claimed tickets

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int N = p.N, nr = p.nr, L = p.L;
    const int nbox = N / 64;
    // the next chunk's inputs go into regions as soon as this chunk is done with them:
    // x, dy and the entering state after phase C, B and C after the unfold's token loop
    auto issue_xs = [&](int item) {
        const ChunkItem it = chunk_item_rcs(p, item);
        const int t0_ = it.c * Q;
        const long long u_ = bhc(p, it.b, it.h, it.c);
        mbar_expect_tx(&bar_in[0], (uint32_t)(2 * Q * PD * 2) + 2 * TILE_BYTES);
        tma_load_4d(sm + fuk::SM_X, &tmX, &bar_in[0], 0, it.h, t0_, it.b);
        tma_load_4d(sm + fuk::SM_DY, &tmDY, &bar_in[0], 0, it.h, t0_, it.b);
        bulk_load(sm + fuk::SM_KT, p.ws_kp + u_ * SLOT_FLOATS, 2 * TILE_BYTES, &bar_in[0]);
    };
    auto issue_bc = [&](int item) {
        const ChunkItem it = chunk_item_rcs(p, item);
        const int t0_ = it.c * Q, g_ = it.h / p.hpg;
        mbar_expect_tx(&bar_in[1], (uint32_t)(2 * Q * N * 2));
        for (int k = 0; k < nbox; ++k) {
            tma_load_4d(sm + fuk::SM_B + k * 8192, &tmB, &bar_in[1], 64 * k, g_, t0_, it.b);
            tma_load_4d(sm + fuk::SM_C + k * 8192, &tmC, &bar_in[1], 64 * k, g_, t0_, it.b);
        }
    };

    // phases issued / completed on each mbarrier (counted by thread 0, which issues
    // every load and the first MMA batch of a phase), for the drain of a CTA that stops
    PhaseCount pc_in[2] = {{0u, 0u}, {0u, 0u}}, pc_m[3] = {{0u, 0u}, {0u, 0u}, {0u, 0u}};
    if (tid == 0) {
        mbar_init(&bar_in[0], 1);
        mbar_init(&bar_in[1], 1);
        mbar_init(&bar_mma[0], 1);
        mbar_init(&bar_mma[1], 2);   // two issuing threads commit phase B
        mbar_init(&bar_mma[2], 1);
        mbar_fence_init();
        tma_prefetch_desc(&tmX);
        tma_prefetch_desc(&tmB);
        tma_prefetch_desc(&tmC);
        tma_prefetch_desc(&tmDY);
        const int first = atomicAdd(chain_ticket(p), 1);   // < nitems: the grid is <= nitems
        s_item[0] = first;
        issue_xs(first);
        ++pc_in[0].issued;
        issue_bc(first);
        ++pc_in[1].issued;
    }
    if (warp == 0) tmem_alloc(tslot, fuk::TMEM_COLS);
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    int item = s_item[0];
    TokPrefetch tok;
    ModePrefetch mp;
    {
        const ChunkItem it = chunk_item_rcs(p, item);
        tok = tok_load(p, it.b, it.h, it.c * Q);
        mp = mode_load(p, it.h);
    }
    const uint32_t tbase = *tslot;
    const uint32_t t_v = tbase, t_v2 = tbase + 64u, t_g = tbase + 128u;
    const int cn = 32 * (warp & 3) + lane, ccq = warp >> 2;   // chain step: row, 16-column block
    bool aborted = false;

    for (int kit = 0; item < nitems; ++kit) {
        // the item after this one (read by every thread after the next barrier)
        if (tid == 0) s_item[1] = atomicAdd(chain_ticket(p), 1);
        const ChunkItem it = chunk_item_rcs(p, item);
        const int c = it.c, h = it.h, b = it.b;
        const int g = h / p.hpg;
        const int t0 = c * Q;
        const long long u = bhc(p, b, h, c);
        const int bh = b * p.H + h, rr = p.nc - 1 - c;   // chunks of (b, h) walked before this one
        const uint32_t par = (uint32_t)(kit & 1);
        mode_rates_from(p, f32, mp);
        chunk_tokens_from(p, f32, t0, tok, true);
        if constexpr (TOK) chunk_angles(p, f32, b, h, t0);
        const int next = s_item[1];
        if (next < nitems) {
            const ChunkItem nx = chunk_item_rcs(p, next);
            tok = tok_load(p, nx.b, nx.h, nx.c * Q);
            mp = mode_load(p, nx.h);
        }
        chunk_mode_constants<TOK>(p, f32);
        const bool ok0 = mbar_wait(&bar_in[0], par, WAIT_LIMIT);
        const bool ok1 = ok0 && mbar_wait(&bar_in[1], par, WAIT_LIMIT);
        if (tid == 0) {
            pc_in[0].done += ok0 ? 1u : 0u;
            pc_in[1].done += ok1 ? 1u : 0u;
        }
        int ok = ok1 ? 1 : 0;
        if (!ok) {
            rev_raise_error(1);
            chain_abort(p);
        }
        if (!__syncthreads_and(ok)) {
            aborted = true;
            break;
        }
        // ---- Bo (B at its sub-block's start) and Cm (C at its sub-block's end), hi + lo
        {
            const int t = tid & 63, grp = tid >> 6;
            const int kb = t >> 4;
            const float St = f32[F_S + t];
            const float dsb = St - (kb == 0 ? 0.f : f32[F_S + 16 * kb - 1]);   // >= 0
            const float dse = St - f32[F_S + 16 * kb + 15];                     // <= 0
            // the write's scale: sigma_t, or per mode Z (ZOH, applied to b below)
            const float sig = ZOH ? 1.f : f32[F_SIG + t];
            const unsigned char *sB = sm + fuk::SM_B, *sC = sm + fuk::SM_C;
            float corr = 0.f;
#pragma unroll 1
            for (int k = 0; k < NP / (8 * fuk::RG); ++k) {
                const int r0 = 8 * (grp + fuk::RG * k);
                if (r0 >= N) break;
                float rc[8], rb[8], vb[8], vc[8];
                ld_rows8(sC, t, r0, rc);
                ld_rows8(sB, t, r0, rb);
#pragma unroll
                for (int j = 0; j < 8; j += 2) {
                    const int r = r0 + j;
                    corr = fmaf(rc[j], rb[j], fmaf(rc[j + 1], rb[j + 1], corr));
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
                        const float a0 = f32[F_A2 + r], a1 = f32[F_A2 + r + 1];
                        vb[j] = sig * rb[j] * ex2_fast(fminf(-a0 * dsb, 120.f));
                        vb[j + 1] = sig * rb[j + 1] * ex2_fast(fminf(-a1 * dsb, 120.f));
                        vc[j] = rc[j] * ex2_fast(fminf(a0 * dse, 120.f));
                        vc[j + 1] = rc[j + 1] * ex2_fast(fminf(a1 * dse, 120.f));
                    } else {
                        const int m = nr + ((r - nr) >> 1);
                        const float a = f32[F_A2 + m], w = f32[F_W + m];
                        float sn, cs;
                        pair_sincos<TOK>(pair_angle<TOK>(f32, m - nr, w, dsb, t, 16 * kb - 1), &sn, &cs);
                        const float eb = sig * ex2_fast(fminf(-a * dsb, 120.f));
                        vb[j] = eb * fmaf(rb[j], cs, rb[j + 1] * sn);
                        vb[j + 1] = eb * fmaf(rb[j + 1], cs, -rb[j] * sn);
                        pair_sincos<TOK>(pair_angle<TOK>(f32, m - nr, w, dse, t, 16 * kb + 15), &sn, &cs);
                        const float ec = ex2_fast(fminf(a * dse, 120.f));
                        vc[j] = ec * fmaf(rc[j], cs, rc[j + 1] * sn);
                        vc[j + 1] = ec * fmaf(rc[j + 1], cs, -rc[j] * sn);
                    }
                }
                const uint32_t off = off_kmaj(t, r0, KM_LBO, KM_SBO);
                st16_split(sm + fuk::SM_BO, sm + fuk::SM_BOL, off, vb);
                st16_split(sm + fuk::SM_CM, sm + fuk::SM_CML, off, vc);
            }
            reinterpret_cast<float *>(sm + fuk::SM_GM)[grp * 64 + t] = corr;   // G tiles come later
        }
        fence_proxy_async();
        fence_before_sync();
        __syncthreads();

        // ---- phase A: V = K_prev dY^T (hi + lo), G = dY X^T ---------------------
        if (tid == 0) {
            fence_after_sync();
            const uint32_t x_base = smem_u32(sm + fuk::SM_X), dy_base = smem_u32(sm + fuk::SM_DY);
            const uint32_t id_v = idesc_bf16(128, 64, false, false);
            for (int part = 0; part < 2; ++part) {
                const uint32_t kt_base = smem_u32(sm + (part ? fuk::SM_KTL : fuk::SM_KT));
                for (int s = 0; s < PD / 16; ++s)
                    mma_bf16(t_v, sdesc(kt_base + s * 256u, 128u, 1024u, LAYOUT_NONE),
                             sdesc(dy_base + s * 32u, 16u, 1024u, LAYOUT_SW128), id_v,
                             part > 0 || s > 0);
            }
            const uint32_t id_g = idesc_bf16(64, 64, false, false);
            for (int s = 0; s < PD / 16; ++s)
                mma_bf16(t_g, sdesc(dy_base + s * 32u, 16u, 1024u, LAYOUT_SW128),
                         sdesc(x_base + s * 32u, 16u, 1024u, LAYOUT_SW128), id_g, s > 0);
            mma_commit(&bar_mma[0]);
            ++pc_m[0].issued;
        }
        if (tid < 64) {
            float cs = 0.f;
#pragma unroll
            for (int k = 0; k < fuk::RG; ++k)
                cs += reinterpret_cast<const float *>(sm + fuk::SM_GM)[k * 64 + tid];
            f32[F_CORR + tid] = cs;   // C_t . B_t
        }
        ok = mbar_wait(&bar_mma[0], par, WAIT_LIMIT) ? 1 : 0;
        if (tid == 0) pc_m[0].done += (uint32_t)ok;
        if (!ok) {
            rev_raise_error(1);
            chain_abort(p);
        }
        fence_after_sync();
        if (!__syncthreads_and(ok)) {
            aborted = true;
            break;
        }
        if (warp >= 4 && warp < 12) {
            // ---- masked G (s <= t) -> four 16-row tiles (rows t, K = s); dy_t . u_t
            const int qd = warp & 3, i0 = 2 * ((warp - 4) >> 2);   // two warps per lane quarter
            for (int i = i0; i < i0 + 2; ++i) {
                float v[16];
                tmem_ld16(tmem_addr(t_g, 32u * qd, 16u * i), v);
                if (lane < 16 && i <= qd) {
                    const int t = 16 * qd + lane;
                    float lo[8], hi[8];
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        lo[j] = (16 * i + j <= t) ? v[j] : 0.f;
                        hi[j] = (16 * i + 8 + j <= t) ? v[8 + j] : 0.f;
                    }
                    unsigned char *gt = sm + fuk::SM_GM + qd * 2048;
                    unsigned char *gl = sm + fuk::SM_GML + qd * 2048;
                    st16_split(gt, gl, off_kmaj(lane, 16 * i, 128u, 1024u), lo);
                    st16_split(gt, gl, off_kmaj(lane, 16 * i + 8, 128u, 1024u), hi);
                    if (i == qd) {
                        float dg = 0.f;
#pragma unroll
                        for (int j = 0; j < 16; ++j)
                            if (j == lane) dg = v[j];
                        f32[F_LAM + t] = dg;   // <dy_t, u_t> (lambda is no longer needed)
                    }
                }
            }
        } else {
            // ---- Ch_t = c_t conj(e^{lam S_t}) = Cm_t conj(F[0][k+1]) (t in sub-block k),
            // hi + lo, into the Gc tiles' place (the carried adjoint arrives later)
            const int th = (warp < 4 ? warp : warp - 8) * 32 + lane;
            for (int pc = th; pc < 64 * (N / 8); pc += 256) {
                const int t = pc & 63, r0 = 8 * (pc >> 6), kb = t >> 4;
                const uint32_t off = off_kmaj(t, r0, KM_LBO, KM_SBO);
                const uint4 hq = *reinterpret_cast<const uint4 *>(sm + fuk::SM_CM + off);
                const uint4 lq = *reinterpret_cast<const uint4 *>(sm + fuk::SM_CML + off);
                const uint32_t hw[4] = {hq.x, hq.y, hq.z, hq.w}, lw[4] = {lq.x, lq.y, lq.z, lq.w};
                const float *fre = f32 + F_KRE + fslot(0, kb + 1) * NP;
                const float *fim = f32 + F_KIM + fslot(0, kb + 1) * NP;
                float v[8];
#pragma unroll
                for (int w2 = 0; w2 < 4; ++w2) {
                    const float2 a2_ = bf2_to_f2(hw[w2]), l2_ = bf2_to_f2(lw[w2]);
                    const float a = a2_.x + l2_.x, d = a2_.y + l2_.y;   // rows r0 + 2 w2, + 1
                    const int r = r0 + 2 * w2;
                    if (r < nr) {
                        v[2 * w2] = a * fre[r];
                        v[2 * w2 + 1] = d * fre[r + 1];
                    } else {   // (a + i d) conj(fr + i fi)
                        const int m = nr + ((r - nr) >> 1);
                        v[2 * w2] = fmaf(a, fre[m], d * fim[m]);
                        v[2 * w2 + 1] = fmaf(d, fre[m], -a * fim[m]);
                    }
                }
                st16_split(sm + fuk::SM_GC, sm + fuk::SM_GCL, off, v);
            }
        }
        // the adjoint carried into this chunk is published by the item of chunk c + 1
        int cw = 1;
        if (tid == 0 && rr > 0 &&
            !wait_count(p.ws_flag + bh, rr, chain_abort_word(p), p.wait_limit)) {
            rev_raise_error(2);
            chain_abort(p);
            cw = 0;
        }
        fence_proxy_async();
        fence_before_sync();
        // also orders the wait before every thread's loads of Gc_c
        if (!__syncthreads_and(cw)) {
            aborted = true;
            break;
        }
        float gcv[16];     // Gc_c of row cn, columns 16 ccq ..; in flight during phase B
#pragma unroll
        for (int j4 = 0; j4 < 4; ++j4) {
            float4 a4 = make_float4(0.f, 0.f, 0.f, 0.f);
            if (rr > 0 && cn < N) a4 = __ldcg(carry_ptr(p, rr & 1, bh, ccq, cn) + j4 * NP);
            gcv[4 * j4] = a4.x;
            gcv[4 * j4 + 1] = a4.y;
            gcv[4 * j4 + 2] = a4.z;
            gcv[4 * j4 + 3] = a4.w;
        }

        // ---- phase B: D_{i,k}, E_{j,k} (hi*hi + hi*lo + lo*hi), Ghat = Ch^T dY ------
        if (tid == 0) {
            fence_after_sync();
            const uint32_t id_d = idesc_bf16(128, 16, true, false);
            const uint32_t bo_off[3] = {fuk::SM_BO, fuk::SM_BO, fuk::SM_BOL};
            const uint32_t g_off[3] = {fuk::SM_GM, fuk::SM_GML, fuk::SM_GM};
            for (int i = 0; i < NSB; ++i)
                for (int k = 0; k <= i; ++k)
                    for (int part = 0; part < 3; ++part)
                        mma_bf16(tbase + d_col(i, k),
                                 sdesc(smem_u32(sm + bo_off[part]) + k * 4096u, 2048u, 128u,
                                       LAYOUT_NONE),
                                 sdesc(smem_u32(sm + g_off[part]) + i * 2048u + k * 256u, 128u,
                                       1024u, LAYOUT_NONE),
                                 id_d, part > 0);
            mma_commit(&bar_mma[1]);
            ++pc_m[1].issued;
        } else if (tid == 32) {
            fence_after_sync();
            const uint32_t id_e = idesc_bf16(128, 16, true, true);
            const uint32_t cm_off3[3] = {fuk::SM_CM, fuk::SM_CM, fuk::SM_CML};
            const uint32_t g_off[3] = {fuk::SM_GM, fuk::SM_GML, fuk::SM_GM};
            for (int j = 0; j < NSB; ++j)
                for (int k = j; k < NSB; ++k)
                    for (int part = 0; part < 3; ++part)
                        mma_bf16(tbase + e_col(j, k),
                                 sdesc(smem_u32(sm + cm_off3[part]) + k * 4096u, 2048u, 128u,
                                       LAYOUT_NONE),
                                 sdesc(smem_u32(sm + g_off[part]) + k * 2048u + j * 256u, 1024u,
                                       128u, LAYOUT_NONE),
                                 id_e, part > 0);
            // Ghat (M = 128 state rows, N = 64 p) into G's columns, which masking has read
            const uint32_t dy_base = smem_u32(sm + fuk::SM_DY);
            const uint32_t id_h = idesc_bf16(128, 64, true, true);
            for (int part = 0; part < 2; ++part) {
                const uint32_t ch_base = smem_u32(sm + (part ? fuk::SM_GCL : fuk::SM_GC));
                for (int s = 0; s < Q / 16; ++s)
                    mma_bf16(t_g, sdesc(ch_base + s * 4096u, 2048u, 128u, LAYOUT_NONE),
                             sdesc(dy_base + s * 2048u, 8192u, 1024u, LAYOUT_SW128), id_h,
                             part > 0 || s > 0);
            }
            mma_commit(&bar_mma[1]);
        }
        ok = mbar_wait(&bar_mma[1], par, WAIT_LIMIT) ? 1 : 0;
        if (tid == 0) pc_m[1].done += (uint32_t)ok;
        if (!ok) {
            rev_raise_error(1);
            chain_abort(p);
        }
        fence_after_sync();
        if (!__syncthreads_and(ok)) {
            aborted = true;
            break;
        }
        // ---- chain step: Gc_c tiles, Gc_{c-1} = conj(E_c) Gc_c + Ghat_c, boundary value --
        {
            const bool c_valid = cn < N, c_pair = c_valid && cn >= nr;
            const bool c_im = c_pair && ((cn - nr) & 1);
            float ghv[16];
            tmem_ld16(tmem_addr(t_g, 32u * (warp & 3), 16u * ccq), ghv);
            // Gc_c as hi / lo operand tiles: shared memory (for V2) and the chunk's slot (for dx)
            unsigned char *slot = reinterpret_cast<unsigned char *>(p.ws_gc + u * SLOT_FLOATS);
#pragma unroll
            for (int g8 = 0; g8 < 2; ++g8) {
                const uint32_t off = off_kmaj(cn, 16 * ccq + 8 * g8, 128u, 1024u);
                float hi[8], lo[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const float v = gcv[8 * g8 + j];
                    hi[j] = __bfloat162float(__float2bfloat16_rn(v));
                    lo[j] = v - hi[j];
                }
                st16(sm + fuk::SM_GC, off, hi);
                st16(sm + fuk::SM_GCL, off, lo);
                st16(slot, off, hi);
                st16(slot + TILE_BYTES, off, lo);
            }
            const int m = c_pair ? nr + ((cn - nr) >> 1) : (c_valid ? cn : 0);
            const float er = f32[F_KRE + fslot(0, 4) * NP + m];
            const float ei = c_pair ? f32[F_KIM + fslot(0, 4) * NP + m] : 0.f;
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const float other = __shfl_xor_sync(0xffffffffu, gcv[j], 1);
                if (!c_valid)
                    gcv[j] = 0.f;
                else if (!c_pair)
                    gcv[j] = fmaf(er, gcv[j], ghv[j]);
                else if (!c_im)   // conj(er + i ei)(a + i d) + Ghat, own row = re
                    gcv[j] = fmaf(er, gcv[j], fmaf(ei, other, ghv[j]));
                else              // own row = im
                    gcv[j] = fmaf(er, gcv[j], fmaf(-ei, other, ghv[j]));
            }
            if (c > 0) {
                float4 *dst = carry_ptr(p, (rr + 1) & 1, bh, ccq, cn);
#pragma unroll
                for (int j4 = 0; j4 < 4; ++j4)
                    __stcg(dst + j4 * NP, make_float4(gcv[4 * j4], gcv[4 * j4 + 1], gcv[4 * j4 + 2],
                                                      gcv[4 * j4 + 3]));
                if (p.ws_qb) {
                    // exact boundary value sum_p conj(Gc_{c-1}) K_end_{c-1} of the decay-gradient
                    // scan (K_end_{c-1} = the state entering this chunk, hi + lo tiles); each
                    // 16-column block writes its own partial slot
                    float kv[16];
#pragma unroll
                    for (int g8 = 0; g8 < 2; ++g8) {
                        const uint32_t off = off_kmaj(cn, 16 * ccq + 8 * g8, 128u, 1024u);
                        const uint4 hq = *reinterpret_cast<const uint4 *>(sm + fuk::SM_KT + off);
                        const uint4 lq = *reinterpret_cast<const uint4 *>(sm + fuk::SM_KTL + off);
                        const uint32_t hw[4] = {hq.x, hq.y, hq.z, hq.w};
                        const uint32_t lw[4] = {lq.x, lq.y, lq.z, lq.w};
#pragma unroll
                        for (int w2 = 0; w2 < 4; ++w2) {
                            const float2 a2_ = bf2_to_f2(hw[w2]), l2_ = bf2_to_f2(lw[w2]);
                            kv[8 * g8 + 2 * w2] = a2_.x + l2_.x;
                            kv[8 * g8 + 2 * w2 + 1] = a2_.y + l2_.y;
                        }
                    }
                    float q = 0.f;
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const float og = __shfl_xor_sync(0xffffffffu, gcv[j], 1);
                        const float ok_ = __shfl_xor_sync(0xffffffffu, kv[j], 1);
                        if (!c_pair)
                            q = fmaf(gcv[j], kv[j], q);
                        else if (!c_im)   // a ka + d kd
                            q = fmaf(gcv[j], kv[j], fmaf(og, ok_, q));
                        else              // a kd - d ka
                            q = fmaf(og, kv[j], fmaf(-gcv[j], ok_, q));
                    }
                    if (c_valid) p.ws_qb[u * 4 * N + ccq * N + cn] = q;
                }
            } else {
                // carry out of the first chunk = dL/dK_{-1}: dh0, dw0 = beta_0 dh0,
                // dbeta_0 = <dh0, w0>
                float beta0 = 0.f;
                if (p.two_ep)
                    beta0 = (1.f - ld_io(p.lam, ix_lam(p, b, 0, h), 1)) * ld_io(p.dt, ix_dt(p, b, 0, h), 1);
                float db0 = 0.f;
                if (c_valid) {
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const long long i0 = ix_st(p, b, h, cn, 16 * ccq + j);
                        if (p.dh0) p.dh0[i0] = gcv[j];
                        if (p.dw0) p.dw0[i0] = beta0 * gcv[j];
                        if (p.w0) db0 = fmaf(gcv[j], p.w0[i0], db0);
                    }
                }
#pragma unroll
                for (int o = 16; o >= 1; o >>= 1) db0 += __shfl_xor_sync(0xffffffffu, db0, o);
                if (lane == 0) f32[F_CP + warp] = db0;   // summed after the next barrier
            }
        }
        fence_proxy_async();
        fence_before_sync();
        __syncthreads();
        // ---- phase C: V2 = Gc_c X^T (hi + lo) ------------------------------------
        if (tid == 0) {
            fence_after_sync();
            const uint32_t x_base = smem_u32(sm + fuk::SM_X);
            const uint32_t id_v = idesc_bf16(128, 64, false, false);
            for (int part = 0; part < 2; ++part) {
                const uint32_t gc_base = smem_u32(sm + (part ? fuk::SM_GCL : fuk::SM_GC));
                for (int s = 0; s < PD / 16; ++s)
                    mma_bf16(t_v2, sdesc(gc_base + s * 256u, 128u, 1024u, LAYOUT_NONE),
                             sdesc(x_base + s * 32u, 16u, 1024u, LAYOUT_SW128), id_v,
                             part > 0 || s > 0);
            }
            mma_commit(&bar_mma[2]);
            ++pc_m[2].issued;
        } else if (tid == fuk::THREADS - 32) {
            // the carry of chunk c - 1 is in place: let its item go (off the issue path)
            if (c > 0) publish_count(p.ws_flag + bh, rr + 1);
            if (c == 0) {
                float acc = 0.f;
                for (int k = 0; k < fuk::THREADS / 32; ++k) acc += f32[F_CP + k];
                p.ws_par[((long long)b * p.H + h) * npar_of(p) + p.ndec + p.np + 1] = acc;
            }
        }
        ok = mbar_wait(&bar_mma[2], par, WAIT_LIMIT) ? 1 : 0;
        if (tid == 0) pc_m[2].done += (uint32_t)ok;
        if (!ok) {
            rev_raise_error(1);
            chain_abort(p);
        }
        fence_after_sync();
        if (!__syncthreads_and(ok)) {
            aborted = true;
            break;
        }
        // the tensor cores and the boundary value are done with x, dy and the entering
        // state: fetch the next chunk's
        if (tid == 0 && next < nitems) {
            issue_xs(next);
            ++pc_in[0].issued;
        }
        // ---- unfold: thread (row n, sub-block i) -----------------------------
        float *red = reinterpret_cast<float *>(sm + fuk::SM_RED);    // [128][RED_LD] B . gbu
        float *red2 = reinterpret_cast<float *>(sm + fuk::SM_RED2);  // [128][RED_LD] ddt terms
        float *xch = reinterpret_cast<float *>(sm + fuk::SM_XCH);    // group totals, partials
        const int n = tid & 127, i = tid >> 7, qd = warp & 3;
        const bool valid = n < N;
        const int m = n < nr ? n : nr + ((n - nr) >> 1);
        const bool pr_row = valid && n >= nr;
        const bool im_row = pr_row && ((n - nr) & 1);
        const float a2 = valid ? f32[F_A2 + m] : 0.f, w = valid ? f32[F_W + m] : 0.f;
        const int jp = pr_row ? (n - nr) >> 1 : 0;   // rotation pair of the row
        const int tc = 16 * i;

        // part 1: dCK_t = e^{lam S_t} V + e^{lam (S_t - Sb_i)} sum_k F[k][i] D_{i,k}
        float kk[16];
        {
            float vv[16], dd[16];
            tmem_ld16(tmem_addr(t_v, 32u * qd, (uint32_t)tc), vv);
            tmem_ld16(tmem_addr(tbase + d_col(i, i), 32u * qd, 0u), dd);
            for (int k = 0; k < i; ++k) {
                float ek[16];
                tmem_ld16(tmem_addr(tbase + d_col(i, k), 32u * qd, 0u), ek);
                const float fr = valid ? f32[F_KRE + fslot(k, i) * NP + m] : 0.f;
                const float fi = valid ? f32[F_KIM + fslot(k, i) * NP + m] : 0.f;
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const float other = __shfl_xor_sync(0xffffffffu, ek[j], 1);
                    // own component of (fr + i fi)(re + i im)
                    dd[j] = pr_row ? fmaf(fr, ek[j], fmaf(im_row ? fi : -fi, other, dd[j]))
                                   : fmaf(fr, ek[j], dd[j]);
                }
            }
            const float Sb = i == 0 ? 0.f : f32[F_S + 16 * i - 1];
            float fr = 1.f, fi = 0.f;   // F[0][i] = e^{lam Sb_i}
            if (i && valid) {
                fr = f32[F_KRE + gslot(i) * NP + m];
                fi = -f32[F_KIM + gslot(i) * NP + m];
            }
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const float ds = f32[F_S + tc + j] - Sb;
                const float mag = ex2_fast(a2 * ds);
                float er = mag, ei = 0.f;
                if (pr_row) {
                    float sn, cs;
                    pair_sincos<TOK>(pair_angle<TOK>(f32, jp, w, ds, tc + j, 16 * i - 1), &sn, &cs);
                    er = mag * cs;
                    ei = mag * sn;
                }
                float Er, Ei;
                cmul(er, ei, fr, fi, Er, Ei);
                const float vo = __shfl_xor_sync(0xffffffffu, vv[j], 1);
                const float dO = __shfl_xor_sync(0xffffffffu, dd[j], 1);
                if (!pr_row)
                    kk[j] = fmaf(Er, vv[j], er * dd[j]);
                else if (!im_row)
                    kk[j] = Er * vv[j] - Ei * vo + er * dd[j] - ei * dO;
                else
                    kk[j] = Ei * vo + Er * vv[j] + ei * dO + er * dd[j];
            }
        }

        // part 2: gbu, the decay-gradient suffix sums, dB / dC, walking backwards
        // per token and row: the ddt term of the suffix sum (a for the decay, -w for the
        // angle); with per-token angles the imaginary rows keep -(suffix sum), the angle's
        // own gradient, which leaves through dtheta instead
        const float coef = !valid ? 0.f
                                  : (im_row ? (TOK ? -1.f : -w) : a2 * 0.6931471805599453f);
        const bool one_head = p.hpg == 1;
        const long long tstride = (long long)p.H * p.N;
        float *gdst = p.ws_gbu + ix_wsk(p, b, t0, h, 0, 1, valid ? n : 0);
        float *cdst = p.ws_dC + ix_wsk(p, b, t0, h, 0, 1, valid ? n : 0);
        const unsigned char *sB = sm + fuk::SM_B, *sC = sm + fuk::SM_C;
        unsigned char *sBw = sm + fuk::SM_B, *sCw = sm + fuk::SM_C;
        float cum = 0.f, dacc = 0.f, sdt = 0.f;
        {
            float vv[16], ee[16];
            tmem_ld16(tmem_addr(t_v2, 32u * qd, (uint32_t)tc), vv);
            tmem_ld16(tmem_addr(tbase + e_col(i, i), 32u * qd, 0u), ee);
            for (int k = i + 1; k < NSB; ++k) {
                float ek[16];
                tmem_ld16(tmem_addr(tbase + e_col(i, k), 32u * qd, 0u), ek);
                const float f2r = valid ? f32[F_KRE + fslot(i + 1, k + 1) * NP + m] : 0.f;
                const float f2i = valid ? f32[F_KIM + fslot(i + 1, k + 1) * NP + m] : 0.f;
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const float other = __shfl_xor_sync(0xffffffffu, ek[j], 1);
                    // own component of (f2r - i f2i)(re + i im)
                    ee[j] = pr_row ? fmaf(f2r, ek[j], fmaf(im_row ? -f2i : f2i, other, ee[j]))
                                   : fmaf(f2r, ek[j], ee[j]);
                }
            }
            const float se = f32[F_S + tc + 15];
            float fr = 1.f, fi = 0.f;   // F[i+1][4]
            if (i < 3 && valid) {
                fr = f32[F_KRE + fslot(i + 1, 4) * NP + m];
                fi = f32[F_KIM + fslot(i + 1, 4) * NP + m];
            }
#pragma unroll
            for (int j = 15; j >= 0; --j) {
                const int t = tc + j;
                const float ds = se - f32[F_S + t];   // >= 0
                const float mag = ex2_fast(a2 * ds);
                float er = mag, ei = 0.f;
                if (pr_row) {
                    float sn, cs;
                    pair_sincos<TOK>(pair_angle<TOK>(f32, jp, w, ds, tc + 15, t), &sn, &cs);
                    er = mag * cs;
                    ei = mag * sn;
                }
                const float vo = __shfl_xor_sync(0xffffffffu, vv[j], 1);
                const float eo = __shfl_xor_sync(0xffffffffu, ee[j], 1);
                float res;
                if (!pr_row) {
                    res = er * fmaf(fr, vv[j], ee[j]);
                } else {
                    // own row is re (im_row false) or im; W = conj(F) V2 + E
                    const float vr = im_row ? vo : vv[j], vi = im_row ? vv[j] : vo;
                    const float e_r = im_row ? eo : ee[j], e_i = im_row ? ee[j] : eo;
                    const float wr = fmaf(fr, vr, fmaf(fi, vi, e_r));
                    const float wi = fmaf(fr, vi, fmaf(-fi, vr, e_i));
                    // conj(er + i ei) (wr + i wi)
                    res = im_row ? fmaf(er, wi, -ei * wr) : fmaf(er, wr, ei * wi);
                }
                const bool tv = valid && t0 + t < L;
                const float m2 = f32[F_LAM + t], bn = f32[F_BN + t];
                const float sig = f32[F_SIG + t], dtv = f32[F_DT + t];
                const float bt = ld_row1(sB, t, n), ct = ld_row1(sC, t, n);
                const float k_ = kk[j];                          // dCK_t
                const float dCt = fmaf(-bn * m2, bt, k_);        // dC_t
                const float co = __shfl_xor_sync(0xffffffffu, ct, 1);
                const float ko = __shfl_xor_sync(0xffffffffu, k_, 1);
                const float bo = __shfl_xor_sync(0xffffffffu, bt, 1);
                // gg: the write's adjoint scale applied to gbu (sigma_t, or conj(Z) per mode)
                float gg, zd = 0.f, zw = 0.f;
                if constexpr (ZOH) {
                    // Z = dt phi1(mu), mu = dt a + i phi; the pair's (re, im) of gbu and b
                    const float ro = __shfl_xor_sync(0xffffffffu, res, 1);
                    const float g_r = im_row ? ro : res, g_i = im_row ? res : ro;
                    const float b_r = im_row ? bo : bt, b_i = im_row ? bt : bo;
                    const float an = a2 * 0.6931471805599453f;
                    const float ph = pr_row ? tok_angle<TOK>(f32, jp, w, t) : 0.f;
                    float f1r, f1i = 0.f, fdr, fdi = 0.f;
                    if (pr_row)   // (a warp holds rows of one kind: no divergence)
                        zoh_phi(dtv * an, ph, f1r, f1i, fdr, fdi);
                    else
                        zoh_phi_real(dtv * an, f1r, fdr);
                    const float zr = dtv * f1r, zi = dtv * f1i;
                    gg = !pr_row ? zr * res : (im_row ? fmaf(-zi, g_r, zr * g_i) : fmaf(zr, g_r, zi * g_i));
                    // dL/dZ = (Re s, -Im s), s = b conj(gbu); it reaches dt through
                    // dZ/d dt, a through dt^2 phi1' and the angle through i dt^2 phi1'
                    // (i dt phi1' for a per-token angle)
                    const float gzr = pr_row ? fmaf(b_r, g_r, b_i * g_i) : bt * res;
                    const float gzi = pr_row ? fmaf(b_r, g_i, -b_i * g_r) : 0.f;
                    float zdr, zdi;
                    if (TOK && pr_row) {   // phi1 + dt a phi1'
                        zdr = fmaf(dtv * an, fdr, f1r);
                        zdi = fmaf(dtv * an, fdi, f1i);
                    } else {               // e^mu = 1 + mu phi1, mu = dt a + i phi
                        const float mr = dtv * an;
                        zdr = 1.f + fmaf(mr, f1r, -ph * f1i);
                        zdi = fmaf(mr, f1i, ph * f1r);
                    }
                    if (tv && !im_row) {   // once per mode: a real row or a pair's re row
                        zd = fmaf(gzr, zdr, gzi * zdi);
                        dacc = fmaf(dtv * dtv, fmaf(gzr, fdr, gzi * fdi), dacc);
                    } else if (tv) {
                        zw = (TOK ? dtv : dtv * dtv) * fmaf(-gzr, fdi, gzi * fdr);
                        if (!TOK) dacc += zw;   // the pair's angle-gradient partial
                    }
                } else {
                    gg = sig * res;
                }
                const float go = __shfl_xor_sync(0xffffffffu, gg, 1);
                float v;
                if (!pr_row)
                    v = fmaf(ct, k_, -bt * gg);
                else if (!im_row)   // Re(conj(c) k) - Re(b conj(g))
                    v = fmaf(ct, k_, fmaf(co, ko, -fmaf(bt, gg, bo * go)));
                else                // Im(conj(c) k) - Im(b conj(g)), own row = im
                    v = fmaf(co, k_, fmaf(-ct, ko, -fmaf(bt, go, -bo * gg)));
                if (!tv) v = 0.f;
                cum += v;
                dacc = fmaf(dtv, im_row ? -cum : cum, dacc);
                sdt += dtv;
                // ddt terms; with a per-token angle the im row's entry is the angle's gradient
                red2[n * fuk::RED_LD + t] = coef * cum + (ZOH ? (im_row ? (TOK ? zw : 0.f) : zd) : 0.f);
                red[n * fuk::RED_LD + t] = tv ? res * bt : 0.f;
                if (one_head) {
                    // dB / dC replace the (t, n) element of the raw B / C tiles that only this
                    // thread reads; the tiles go out by TMA stores (rows past L are clipped)
                    if (valid) {
                        st_row1(sBw, t, n, fmaf(-bn * ct, m2, gg));
                        st_row1(sCw, t, n, dCt);
                    }
                } else if (tv) {
                    gdst[(long long)t * tstride] = res;
                    cdst[(long long)t * tstride] = dCt;
                }
            }
        }
        // later sub-blocks carry into every token of earlier ones
        xch[i * 128 + n] = cum;
        fence_proxy_async();   // the staged dB / dC tiles are read by TMA stores
        __syncthreads();
        if (tid == 0) {
            if (one_head) {
                for (int k = 0; k < nbox; ++k) {
                    tma_store_4d(&tmDB, sm + fuk::SM_B + k * 8192, 64 * k, g, t0, b);
                    tma_store_4d(&tmDC, sm + fuk::SM_C + k * 8192, 64 * k, g, t0, b);
                }
                bulk_commit();
            } else if (next < nitems) {
                // every token loop is done with the raw B / C tiles: fetch the next chunk's
                issue_bc(next);
                ++pc_in[1].issued;
            }
        }
        float later = 0.f;
        for (int k = i + 1; k < fuk::TQ; ++k) later += xch[k * 128 + n];
        if (later != 0.f) {
            const float add = coef * later;
            for (int t = tc; t < tc + 16; ++t) red2[n * fuk::RED_LD + t] += add;
        }
        if (TOK && im_row) {
            // dL/dtheta_t of this pair, kept out of ddt: the part from inside the chunk and
            // the carry from later chunks, minus the imaginary part of the exact value at
            // the chunk's end boundary (published with the adjoint this item waited for)
            float cai = 0.f;
            if (p.ws_qb && c + 1 < p.nc) {
                const float *q = p.ws_qb + ((long long)bh * p.nc + c + 1) * 4 * (long long)N;
#pragma unroll
                for (int w2 = 0; w2 < 4; ++w2) cai += __ldcg(q + w2 * N + n);
            }
            for (int t = tc; t < tc + 16; ++t) {
                if (t0 + t < L) p.dtheta[ix_th(p, b, t0 + t, h, jp)] = red2[n * fuk::RED_LD + t] - cai;
                red2[n * fuk::RED_LD + t] = 0.f;
            }
        }
        dacc += (im_row ? -later : later) * sdt;
        xch[(fuk::TQ + i) * 128 + n] = dacc;
        __syncthreads();
        if (i == 0 && valid) {
            float tot = 0.f, da = 0.f;
            for (int k = 0; k < fuk::TQ; ++k) {
                tot += xch[k * 128 + n];
                da += xch[(fuk::TQ + k) * 128 + n];
            }
            const int nmode = p.nr + p.np;
            float *blk = p.ws_blk + u * (4 * nmode + 2);
            if (!pr_row) {
                blk[4 * m + 0] = tot;
                blk[4 * m + 1] = 0.f;
                blk[4 * m + 2] = da;
                blk[4 * m + 3] = 0.f;
            } else if (!im_row) {
                blk[4 * m + 0] = tot;
                blk[4 * m + 2] = da;
            } else {
                blk[4 * m + 1] = tot;
                blk[4 * m + 3] = da;
            }
        }
        // column sums over the state rows: all threads, 128 / RG rows each, fixed order
        float *part = xch + 2 * fuk::TQ * 128;   // [2][RG][64]
        {
            const int t = tid & 63, rg = tid >> 6;
            constexpr int RPG = NP / fuk::RG;
            float s1 = 0.f, s2 = 0.f;
            for (int k = rg * RPG; k < rg * RPG + RPG && k < N; ++k) {
                s1 += red[k * fuk::RED_LD + t];
                s2 += red2[k * fuk::RED_LD + t];
            }
            part[rg * 64 + t] = s1;
            part[(fuk::RG + rg) * 64 + t] = s2;
        }
        __syncthreads();
        if (tid == 0 && one_head) {
            // the dB / dC stores have read the B / C tiles: fetch the next chunk's
            bulk_wait_read_all();
            if (next < nitems) {
                issue_bc(next);
                ++pc_in[1].issued;
            }
        }
        if (tid < 64 && t0 + tid < L) {
            const int t = tid;
            float dsig = 0.f, dd = 0.f;
            for (int k = 0; k < fuk::RG; ++k) {
                dsig += part[k * 64 + t];
                dd += part[(fuk::RG + k) * 64 + t];
            }
            const long long ii = ix_bth(p, b, t0 + t, h);
            const float m2 = f32[F_LAM + t];
            p.ws_tok[2 * ii] = dsig;
            p.ws_tok[2 * ii + 1] = f32[F_CORR + t] * m2;
            p.ws_M2[ii] = m2;
            p.ws_ddt[ii] = dd;
        }
        if (warp == 2) {   // the chunk's sum of dt and of <dy_t, u_t>
            float st_ = f32[F_DT + lane] + f32[F_DT + lane + 32];
            float dD = (t0 + lane < L ? f32[F_LAM + lane] : 0.f) +
                       (t0 + lane + 32 < L ? f32[F_LAM + lane + 32] : 0.f);
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1) {
                st_ += __shfl_xor_sync(0xffffffffu, st_, o);
                dD += __shfl_xor_sync(0xffffffffu, dD, o);
            }
            if (lane == 0) {
                const int nmode = p.nr + p.np;
                float *blk = p.ws_blk + u * (4 * nmode + 2);
                blk[4 * nmode + 0] = st_;
                blk[4 * nmode + 1] = (p.O == p.R) ? dD : 0.f;
            }
        }
        fence_before_sync();
        __syncthreads();
        item = next;
    }
    if (aborted && tid == 0) {
        // every load and MMA still in flight lands before the CTA's shared memory and
        // TMEM go away
        drain_phases(&bar_in[0], pc_in[0]);
        drain_phases(&bar_in[1], pc_in[1]);
        for (int q = 0; q < 3; ++q) drain_phases(&bar_mma[q], pc_m[q]);
    }
    if (tid == 0) bulk_wait_read_all();
    fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        fence_after_sync();
        tmem_dealloc(tbase, fuk::TMEM_COLS);
    }
}

}  // namespace chunkrev

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
// Opt-in to the dynamic shared memory of a kernel on the current device (the
// attribute is per device, so the flag is kept per device ordinal).
template <typename K>
static cudaError_t set_smem(K kern, uint32_t bytes, bool (&done)[64]) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64 && done[dev]) return cudaSuccess;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e == cudaSuccess && dev >= 0 && dev < 64) done[dev] = true;
    return e;
}

cudaError_t chunk_states(const Params &p, cudaStream_t st);
int sm_count();

// Shared memory opt-in of the dx and fused kernels of one angle mode and write form.
template <bool TOK, bool ZOH>
static cudaError_t rev_smem() {
    using namespace chunkrev;
    static bool a3[64] = {}, a4[64] = {};
    cudaError_t e;
    if ((e = set_smem(k_chunk_bwd_dx<TOK, ZOH>, dxk::smem_bytes<TOK>(), a3)) != cudaSuccess) return e;
    return set_smem(k_chunk_bwd_fused<TOK, ZOH>, fuk::smem_bytes<TOK>(), a4);
}

// The state entering every chunk for the tensor-core backward (p.ws_kp,
// p.ws_ce), unless the forward's are given (p.states_ready).
cudaError_t chunk_bwd_states(const Params &p, cudaStream_t st) {
    return p.states_ready ? cudaSuccess : chunk_states(p, st);
}

// The rest of the tensor-core backward: the chunk-local adjoints, the reverse
// pass (exact chunk-boundary values, dh0 / dw0 / dbeta_0), dx, and the fused
// per-chunk kernel (dC, gbu, dsigma, <dy, u>, the within-chunk decay sums, dB
// / dC).  Needs p.ws_kp and p.ws_ce from chunk_bwd_states.
cudaError_t chunk_bwd_reverse(const Params &p, cudaStream_t st) {
    using namespace chunkrev;
    CUtensorMap mx, mb, mc, mdy;
    if (!make_map(&mx, p.x, PD, p.H, p.L, p.Bsz, p.sx[2], p.sx[1], p.sx[0], PD, true) ||
        !make_map(&mb, p.Bm, p.N, p.G, p.L, p.Bsz, p.sB[2], p.sB[1], p.sB[0], 64, true) ||
        !make_map(&mc, p.Cm, p.N, p.G, p.L, p.Bsz, p.sC[2], p.sC[1], p.sC[0], 64, true) ||
        !make_map(&mdy, p.dy, PD, p.H, p.L, p.Bsz, p.sy[2], p.sy[1], p.sy[0], PD, true))
        return cudaErrorInvalidValue;
    if (!p.ws_ring || !p.ws_flag) return cudaErrorInvalidValue;
    cudaError_t e;
    if ((e = by_variant(p, [&](auto tok, auto zoh) {
             return rev_smem<decltype(tok)::value, decltype(zoh)::value>();
         })) != cudaSuccess)
        return e;
    // the per-(b, h) carry counters, the ticket and the abort word start at zero on every call
    if ((e = cudaMemsetAsync(p.ws_flag, 0, sizeof(int) * ((size_t)p.Bsz * p.H + 2), st)) !=
        cudaSuccess)
        return e;
    {
        const long long nitems = (long long)p.nc * p.H * p.Bsz;
        const int pgrid = (int)(nitems < sm_count() ? nitems : sm_count());
        // dB / dC leave the fused kernel by TMA stores when every group has one head
        CUtensorMap mdb = mb, mdc = mc;
        if (p.hpg == 1 &&
            (!make_map(&mdb, p.dBm, p.N, p.G, p.L, p.Bsz, p.sB[2], p.sB[1], p.sB[0], 64, true) ||
             !make_map(&mdc, p.dCm, p.N, p.G, p.L, p.Bsz, p.sC[2], p.sC[1], p.sC[0], 64, true)))
            return cudaErrorInvalidValue;
        by_variant(p, [&](auto tok, auto zoh) {
            constexpr bool T = decltype(tok)::value, Z = decltype(zoh)::value;
            k_chunk_bwd_fused<T, Z>
                <<<pgrid, fuk::THREADS, fuk::smem_bytes<T>(), st>>>(mx, mb, mc, mdy, mdb, mdc, p);
            return cudaSuccess;
        });
    }
    profile_mark(st, "k_chunk_bwd_fused");
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    // dx reads the adjoint carries the fused kernel left in every chunk's slot
    const dim3 grid(p.nc, p.H, p.Bsz);
    if (p.sv_P) {
        static bool a5[64] = {};
        if ((e = set_smem(k_chunk_bwd_dx_saved, dxs::SMEM_BYTES, a5)) != cudaSuccess) return e;
        k_chunk_bwd_dx_saved<<<grid, dxs::THREADS, dxs::SMEM_BYTES, st>>>(mdy, p);
        profile_mark(st, "k_chunk_bwd_dx_saved");
    } else {
        by_variant(p, [&](auto tok, auto zoh) {
            constexpr bool T = decltype(tok)::value, Z = decltype(zoh)::value;
            k_chunk_bwd_dx<T, Z><<<grid, dxk::THREADS, dxk::smem_bytes<T>(), st>>>(mb, mc, mdy, p);
            return cudaSuccess;
        });
        profile_mark(st, "k_chunk_bwd_dx");
    }
    return cudaGetLastError();
}

// Read and clear the device error word of these kernels.
int chunk_rev_error_take() {
    int v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, ssm_chunk_rev_error_word, sizeof(int)) != cudaSuccess) return -1;
    if (v) cudaMemcpyToSymbol(ssm_chunk_rev_error_word, &zero, sizeof(int));
    return v;
}

}  // namespace ssm
