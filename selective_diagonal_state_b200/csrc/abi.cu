// C ABI of the selective diagonal scan library: argument validation, workspace
// sizing, error reporting and dispatch to the kernels.  See include/ssm_scan.h.
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <atomic>
#include <mutex>
#include <string>
#include <vector>

#include "../../include/ssm_scan.h"
#include "common.cuh"

namespace ssm {
bool simt_supported(const Params &p);
cudaError_t simt_forward(const Params &p, cudaStream_t st);
cudaError_t simt_backward(const Params &p, cudaStream_t st);
cudaError_t chunk_backward(const Params &p, cudaStream_t st);
cudaError_t chunk_range_check(const Params &p, int *gate, cudaStream_t st);
bool chunk_bwd_supported(const Params &p);
bool chunk_fwd_supported(const Params &p);
cudaError_t chunk_forward(const Params &p, cudaStream_t st);
cudaError_t chunk_states(const Params &p, cudaStream_t st);
int chunk_error_take();
int chunk_rev_error_take();
bool step_supported(const Params &p);
struct PreactArgs {
    const void *z, *lam_logit, *ddt, *dlam;
    const float *bias;
    void *dt, *lam, *dz, *dlam_logit;
    float *dbias;
};
cudaError_t preact_forward(const Params &p, const PreactArgs &a, cudaStream_t st);
cudaError_t preact_backward(const Params &p, const PreactArgs &a, cudaStream_t st);
cudaError_t scan_step(const Params &p, float *h, float *w, cudaStream_t st);
bool ssd_supported(const Params &p);
int ssd_chunk_tokens(int R);
size_t ssd_ring_bytes(long long B, long long H, long long L, int R);
cudaError_t ssd_forward(const Params &p, cudaStream_t st);
cudaError_t ssd_backward(const Params &p, cudaStream_t st);
int ssd_error_take();
bool m1_supported(const Params &p);
size_t m1_kept_floats(long long B, long long L, long long H, int N);
size_t m1_part_floats(long long B, long long L, long long H, int N);
cudaError_t m1_forward(const Params &p, float *kept, cudaStream_t st);
cudaError_t m1_backward(const Params &p, float *kept, bool kept_ready, float *part,
                        cudaStream_t st);
cudaError_t cp_transition(const Params &p, float *phi, float *beta0, cudaStream_t st);
cudaError_t cp_state_combine(const Params &p, int seg, const float *hT_all, const float *wT_all,
                             const float *phi_all, const float *beta0_all, const float *h0,
                             const float *w0, float *h_in, float *w_in, cudaStream_t st);
cudaError_t cp_adjoint_combine(const Params &p, int nseg, int seg, const float *dh0_all,
                               const float *phi_all, const float *beta0_all, const float *dhT,
                               float *dh_end, float *dw_end, cudaStream_t st);
cudaError_t cp_write_adjoint(const Params &p, const float *dw_end, cudaStream_t st);
cudaError_t cp_fill_tail(const Params &p, int nv, const float *dh_end, cudaStream_t st);
cudaError_t gate_forward(const Params &p, cudaStream_t st);
cudaError_t gate_backward(const Params &p, const void *dyg, void *dy, void *dz, cudaStream_t st);
}  // namespace ssm

namespace {

thread_local std::string g_last_error;

// polls of a carry counter before a chained kernel's wait gives up
std::atomic<long long> g_wait_limit{1ll << 22};

// Gate words of the device-side choice between the tensor-core chain and the
// recurrent chain (written by the range check of each call).  One slot per
// call from a ring, so that calls in flight on different streams do not share
// a word.
constexpr unsigned kGateSlots = 4096;
__device__ int g_gate_ring[kGateSlots];
std::atomic<unsigned> g_gate_next{0};
std::mutex g_gate_mu;
int *g_gate_base[64];
// route of the last call on this host thread: its gate word (chunk-eligible
// calls) or the recurrent route chosen on the host
thread_local const int *g_last_gate = nullptr;
thread_local int g_last_route = -1;

cudaError_t gate_slot(int **out, cudaStream_t st) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    {
        std::lock_guard<std::mutex> lock(g_gate_mu);
        if (!g_gate_base[dev]) {
            void *ptr = nullptr;
            if ((e = cudaGetSymbolAddress(&ptr, g_gate_ring)) != cudaSuccess) return e;
            g_gate_base[dev] = static_cast<int *>(ptr);
        }
    }
    int *g = g_gate_base[dev] + (g_gate_next.fetch_add(1) % kGateSlots);
    if ((e = cudaMemsetAsync(g, 0, sizeof(int), st)) != cudaSuccess) return e;
    *out = g;
    return cudaSuccess;
}

// per-kernel timing session (see ssm_scan_profile_start)
struct ProfileRec {
    const char *name;
    int ev0, ev1;
};
struct ProfileSession {
    bool active = false;
    std::vector<cudaEvent_t> pool;
    size_t used = 0;
    int cur = -1;  // event that opens the next launch of the current call
    std::vector<ProfileRec> recs;
};
thread_local ProfileSession g_prof;

void profile_begin(cudaStream_t st) {
    if (!g_prof.active || g_prof.used >= g_prof.pool.size()) {
        g_prof.cur = -1;
        return;
    }
    cudaEventRecord(g_prof.pool[g_prof.used], st);
    g_prof.cur = (int)g_prof.used++;
}
void profile_end() { g_prof.cur = -1; }

int fail(int code, const char *fmt, ...) __attribute__((format(printf, 2, 3)));
int fail(int code, const char *fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return code;
}

int cuda_fail(cudaError_t e, const char *where) {
    return fail(SSM_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

inline size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

int nstate(const ssm_desc_t *d) { return d->n_real + 2 * d->n_pairs; }
int ndecay(const ssm_desc_t *d) {
    return d->decay_mode == SSM_DECAY_PER_HEAD ? 1 : d->n_real + d->n_pairs;
}

int validate_desc(const ssm_desc_t *d) {
    if (!d) return fail(SSM_ERR_ARG, "descriptor is NULL");
    if (d->batch < 0 || d->seqlen < 0) return fail(SSM_ERR_ARG, "batch and seqlen must be >= 0");
    if (d->nheads < 1 || d->headdim < 1 || d->ngroups < 1)
        return fail(SSM_ERR_ARG, "nheads, headdim and ngroups must be >= 1");
    if (d->nheads % d->ngroups)
        return fail(SSM_ERR_ARG, "nheads (%lld) must be a multiple of ngroups (%lld)",
                    (long long)d->nheads, (long long)d->ngroups);
    if (d->n_real < 0 || d->n_pairs < 0 || nstate(d) < 1)
        return fail(SSM_ERR_ARG, "need n_real >= 0, n_pairs >= 0 and n_real + 2 n_pairs >= 1");
    if (d->rank_in < 1 || d->rank_out < 1) return fail(SSM_ERR_ARG, "rank_in, rank_out must be >= 1");
    if (d->decay_mode != SSM_DECAY_PER_HEAD && d->decay_mode != SSM_DECAY_PER_COORD)
        return fail(SSM_ERR_ARG, "unknown decay_mode %d", d->decay_mode);
    if (d->two_endpoint != 0 && d->two_endpoint != 1)
        return fail(SSM_ERR_ARG, "two_endpoint must be 0 or 1");
    if (d->dtype_io != SSM_F32 && d->dtype_io != SSM_BF16)
        return fail(SSM_ERR_ARG, "unknown dtype_io %d", d->dtype_io);
    if (d->chunk < 0) return fail(SSM_ERR_ARG, "chunk must be >= 0");
    if (d->angle_mode != SSM_ANGLE_STATIC && d->angle_mode != SSM_ANGLE_PER_TOKEN)
        return fail(SSM_ERR_ARG, "unknown angle_mode %d", d->angle_mode);
    if (d->n_static < 0 || d->n_static > d->n_real)
        return fail(SSM_ERR_ARG, "n_static (%d) must lie in [0, n_real = %d]", d->n_static, d->n_real);
    if (d->discretization != SSM_DISC_EULER && d->discretization != SSM_DISC_ZOH)
        return fail(SSM_ERR_ARG, "unknown discretization %d", d->discretization);
    if (d->discretization == SSM_DISC_ZOH && (d->two_endpoint || d->n_static))
        return fail(SSM_ERR_ARG, "the ZOH write needs two_endpoint == 0 and n_static == 0");
    if (d->reserved_ != 0) return fail(SSM_ERR_ARG, "reserved descriptor field must be 0");
    if (d->batch > 65535) return fail(SSM_ERR_UNSUPPORTED, "batch > 65535");
    if (d->seqlen > (1LL << 31) - 1 || d->nheads > (1 << 24) || d->headdim > (1 << 16))
        return fail(SSM_ERR_UNSUPPORTED, "sizes exceed the 32-bit index ranges of the kernels");
    const int64_t *st[] = {d->stride_x, d->stride_y, d->stride_B,
                           d->stride_C, d->stride_dt, d->stride_lambda};
    for (int i = 0; i < 6; ++i)
        for (int k = 0; k < 3; ++k)
            if (st[i][k] < 0) return fail(SSM_ERR_ARG, "negative stride");
    return SSM_OK;
}

int check_ptr(const void *ptr, const char *name, size_t align) {
    if (!ptr) return fail(SSM_ERR_ARG, "%s is NULL", name);
    if ((uintptr_t)ptr % align) return fail(SSM_ERR_ALIGN, "%s is not %zu-byte aligned", name, align);
    return SSM_OK;
}

void fill_params(const ssm_desc_t *d, ssm::Params &p) {
    memset(&p, 0, sizeof(p));
    p.Bsz = (int)d->batch;
    p.L = (int)d->seqlen;
    p.H = (int)d->nheads;
    p.P = (int)d->headdim;
    p.G = (int)d->ngroups;
    p.nr = d->n_real;
    p.np = d->n_pairs;
    p.N = nstate(d);
    p.R = d->rank_in;
    p.O = d->rank_out;
    p.ndec = ndecay(d);
    p.hpg = (int)(d->nheads / d->ngroups);
    p.two_ep = d->two_endpoint;
    p.per_coord = d->decay_mode == SSM_DECAY_PER_COORD;
    p.bf16 = d->dtype_io == SSM_BF16;
    p.angle_tok = d->angle_mode == SSM_ANGLE_PER_TOKEN && d->n_pairs > 0;
    p.nst = d->n_static;
    p.zoh = d->discretization == SSM_DISC_ZOH;
    p.wait_limit = g_wait_limit.load();
    for (int k = 0; k < 3; ++k) {
        p.sx[k] = d->stride_x[k];
        p.sy[k] = d->stride_y[k];
        p.sB[k] = d->stride_B[k];
        p.sC[k] = d->stride_C[k];
        p.sdt[k] = d->stride_dt[k];
        p.slam[k] = d->stride_lambda[k];
    }
}

struct BwdWs {
    size_t off_dC, off_gbu, off_tok, off_M2, off_par, off_ddt, off_blk, off_blkc, off_kp, off_qb,
        off_gc, off_ce, off_ring, off_flag, total;
    bool boundary;  // chunk-boundary carries (tensor-core backward shapes)
};

// Shapes the tensor-core chain may take (pointer alignment is checked at call time).
bool tensor_chain_shape(const ssm_desc_t *d) {
    const int N = d->n_real + 2 * d->n_pairs;
    return d->dtype_io == SSM_BF16 && d->headdim == 64 && d->rank_in == 1 && d->rank_out == 1 &&
           (N == 64 || N == 128) && d->n_real % 8 == 0 && d->chunk != 1 && d->seqlen > 0 &&
           d->n_static == 0;
}

// Shapes of the scalar-decay (per-head) tensor-core chain: Mamba-2 SISO and
// SSD-MIMO with R, O in {1, 2, 4} (pointer alignment is checked at call time).
bool ssd_shape(const ssm_desc_t *d) {
    const int N = d->n_real + 2 * d->n_pairs;
    auto rank_ok = [](int r) { return r == 1 || r == 2 || r == 4; };
    return d->dtype_io == SSM_BF16 && d->decay_mode == SSM_DECAY_PER_HEAD && d->n_pairs == 0 &&
           d->headdim == 64 && (N == 64 || N == 128) && rank_ok(d->rank_in) &&
           rank_ok(d->rank_out) && d->chunk != 1 && d->seqlen > 0 && d->n_static == 0 &&
           d->discretization == SSM_DISC_EULER;
}
// (token, rank) rows per token of the scalar-decay chain: the wider of the two ranks
// (the narrower side's extra rows are zero)
static int ssd_rank(const ssm_desc_t *d) { return d->rank_in > d->rank_out ? d->rank_in : d->rank_out; }

// Shapes of the channel scan (Mamba-1: head dim 1, 8 or 16 real state rows,
// groups of a multiple of 64 channels).
bool m1_shape(const ssm_desc_t *d) {
    const int N = d->n_real + 2 * d->n_pairs;
    return d->dtype_io == SSM_BF16 && d->headdim == 1 && d->rank_in == 1 && d->rank_out == 1 &&
           d->n_pairs == 0 && (N == 8 || N == 16) && (d->nheads / d->ngroups) % 64 == 0 &&
           d->chunk != 1 && d->seqlen > 0 && d->n_static == 0 &&
           d->discretization == SSM_DISC_EULER;
}

// Forward workspace of the tensor-core chain.  Every forward carries the fp32
// state from one 64-token chunk to the next through two 32 KB slots and one
// counter per (b, h) (the first `total_infer` bytes).  A training forward
// (workspace of `total` bytes) also keeps, per chunk, the state entering it
// (bf16 hi + lo tiles, 32 KB), the chunk decays (128 x 2 floats), the masked
// score tiles (8 KB), the chunk-end folded B tile (16 KB) and the diagonal
// correction (64 floats) for ssm_scan_bwd_saved.
struct FwdWs {
    size_t off_ring, off_flag, off_kp, off_ce, off_P, off_Bh, off_corr, total_infer, total;
};
FwdWs fwd_layout(const ssm_desc_t *d) {
    FwdWs w;
    w.off_ring = w.off_flag = w.off_kp = w.off_ce = w.off_P = w.off_Bh = w.off_corr = 0;
    w.total_infer = w.total = 0;
    if (m1_shape(d)) {
        // channel scan: a forward alone needs nothing; a training forward keeps the
        // state entering every 16-token tile
        w.off_kp = 0;
        w.total = align256(ssm::m1_kept_floats(d->batch, d->seqlen, d->nheads, nstate(d)) * 4);
        return w;
    }
    if (ssd_shape(d)) {
        // scalar-decay chain: the chain buffers (segment states and decays, a carry
        // slot per CTA, the backward's adjoint slots), the counters of every (b, h), the
        // ticket and abort words; a training forward also keeps the state entering every
        // chunk of ssm::ssd_chunk_tokens tokens (bf16 hi + lo tiles, 32 KB)
        const size_t bh = (size_t)d->batch * d->nheads;
        const int qt = ssm::ssd_chunk_tokens(ssd_rank(d));
        const size_t units = bh * (size_t)((d->seqlen + qt - 1) / qt);
        const size_t slot = 128 * (size_t)d->headdim * 4;
        size_t off = align256(ssm::ssd_ring_bytes(d->batch, d->nheads, d->seqlen, ssd_rank(d)));
        w.off_flag = off;
        off = align256(off + (bh + 2) * 4);
        w.total_infer = off;
        w.off_kp = off;
        off = align256(off + units * slot);
        w.total = off;
        return w;
    }
    if (!tensor_chain_shape(d)) return w;
    const size_t bh = (size_t)d->batch * d->nheads;
    const size_t units = bh * (size_t)((d->seqlen + 63) / 64);
    const size_t slot = 128 * (size_t)d->headdim * 4;   // 128 state rows x P, fp32 (32 KB)
    // every forward: the two carry slots and the carry counter of each (b, h)
    w.off_ring = 0;
    size_t off = align256(2 * bh * slot);
    w.off_flag = off;   // carry counters, then the work-item ticket and the abort word
    off = align256(off + (bh + 2) * 4);
    w.total_infer = off;
    // a training forward also keeps, per chunk, the state entering it (bf16 hi + lo
    // tiles), the chunk decays and the products the backward reuses
    w.off_kp = off;
    off = align256(off + units * slot);
    w.off_ce = off;
    off = align256(off + units * 128 * 2 * 4);
    w.off_P = off;
    off = align256(off + units * 8192);
    w.off_Bh = off;
    off = align256(off + units * 16384);
    w.off_corr = off;
    off = align256(off + units * 64 * 4);
    w.total = off;
    return w;
}

// Backward workspace of the scalar-decay chain: the adjoint carry slots and
// counters, the entering states of every chunk (unless a training forward's are
// given), per-token and per-chunk sums, and the per-head dB / dC of groups that
// hold several heads.
struct SsdBwdWs {
    size_t off_ring, off_flag, off_kp, off_tok, off_par, off_db0, off_dBh, off_dCh, total;
};
SsdBwdWs ssd_bwd_layout(const ssm_desc_t *d) {
    SsdBwdWs w;
    const size_t bh = (size_t)d->batch * d->nheads;
    const int qt = ssm::ssd_chunk_tokens(ssd_rank(d));
    const size_t nc = (size_t)((d->seqlen + qt - 1) / qt);
    const size_t slot = 128 * (size_t)d->headdim * 4;
    const size_t BLH = (size_t)d->batch * d->seqlen * d->nheads;
    const size_t N = nstate(d);
    size_t off = 0;
    w.off_ring = off;   // carry slots and the forward's segment buffers
    off = align256(off + ssm::ssd_ring_bytes(d->batch, d->nheads, d->seqlen, ssd_rank(d)));
    w.off_flag = off;
    off = align256(off + (bh + 2) * 4);
    w.off_kp = off;
    off = align256(off + bh * nc * slot);
    w.off_tok = off;
    off = align256(off + BLH * 3 * 4);
    w.off_par = off;
    off = align256(off + bh * nc * 2 * 4);
    w.off_db0 = off;
    off = align256(off + bh * 4);
    w.off_dBh = w.off_dCh = off;
    if (d->nheads != d->ngroups) {
        w.off_dBh = off;
        off = align256(off + BLH * d->rank_in * N * 4);
        w.off_dCh = off;
        off = align256(off + BLH * d->rank_out * N * 4);
    }
    w.total = off;
    return w;
}

// Stride conditions of the channel scan and of the scalar-decay chain, which the
// descriptor alone decides (the kernels also need 16-byte aligned tensor bases,
// known only at call time).
bool m1_strides(const ssm_desc_t *d) {
    auto m8 = [](int64_t v) { return v % 8 == 0; };
    bool ok = d->stride_x[2] == 1 && d->stride_y[2] == 1 && d->stride_dt[2] == 1;
    for (int k = 0; k < 2; ++k)
        ok = ok && m8(d->stride_x[k]) && m8(d->stride_y[k]) && m8(d->stride_dt[k]);
    if (d->two_endpoint)
        ok = ok && d->stride_lambda[2] == 1 && m8(d->stride_lambda[0]) && m8(d->stride_lambda[1]);
    for (int k = 0; k < 3; ++k) ok = ok && m8(d->stride_B[k]) && m8(d->stride_C[k]);
    return ok;
}
bool ssd_strides(const ssm_desc_t *d) {
    auto st16 = [](int64_t v) { return (v * 2) % 16 == 0; };
    bool ok = true;
    for (int k = 0; k < 3; ++k)
        ok = ok && st16(d->stride_x[k]) && st16(d->stride_y[k]) && st16(d->stride_B[k]) &&
             st16(d->stride_C[k]);
    return ok;
}
size_t m1_bwd_bytes(const ssm_desc_t *d) {
    return align256(ssm::m1_kept_floats(d->batch, d->seqlen, d->nheads, nstate(d)) * 4) +
           align256(ssm::m1_part_floats(d->batch, d->seqlen, d->nheads, nstate(d)) * 4);
}

BwdWs bwd_layout(const ssm_desc_t *d) {
    BwdWs w;
    const size_t BLH = (size_t)d->batch * d->seqlen * d->nheads;
    const size_t N = nstate(d);
    size_t off = 0;
    w.off_dC = off;
    off = align256(off + BLH * d->rank_out * N * 4);
    w.off_gbu = off;
    off = align256(off + BLH * d->rank_in * N * 4);
    w.off_tok = off;
    off = align256(off + BLH * 2 * 4);
    w.off_M2 = off;
    off = align256(off + BLH * d->rank_out * d->rank_in * 4);
    w.off_par = off;
    off = align256(off + (size_t)d->batch * d->nheads * (ndecay(d) + d->n_pairs + 2) * 4);
    const size_t ntb = (size_t)(d->seqlen + 63) / 64;  // time blocks of the finalize scan
    const size_t nmode = (size_t)d->n_real + d->n_pairs;
    w.off_ddt = off;
    off = align256(off + BLH * 4);
    w.off_blk = off;
    off = align256(off + (size_t)d->batch * d->nheads * ntb * (4 * nmode + 2) * 4);
    w.off_blkc = off;
    off = align256(off + (size_t)d->batch * d->nheads * ntb * 4);
    w.boundary = tensor_chain_shape(d);
    w.off_kp = w.off_qb = w.off_gc = w.off_ce = w.off_ring = w.off_flag = off;
    if (w.boundary) {
        w.off_kp = off;
        off = align256(off + (size_t)d->batch * d->nheads * ntb * 128 * d->headdim * 4);
        w.off_qb = off;
        off = align256(off + (size_t)d->batch * d->nheads * ntb * 4 * N * 4);
        w.off_gc = off;
        off = align256(off + (size_t)d->batch * d->nheads * ntb * 128 * d->headdim * 4);
        w.off_ce = off;
        off = align256(off + (size_t)d->batch * d->nheads * ntb * 128 * 2 * 4);
        // the adjoint carried between chunks: two fp32 slots and a counter per (b, h)
        w.off_ring = off;
        off = align256(off + 2 * (size_t)d->batch * d->nheads * 128 * d->headdim * 4);
        w.off_flag = off;   // carry counters, then the work-item ticket and the abort word
        off = align256(off + ((size_t)d->batch * d->nheads + 2) * 4);
    }
    w.total = off;
    return w;
}

int common_inputs(const ssm_desc_t *d, const void *x, const void *dt, const float *A_log,
                  const float *theta, const void *B, const void *C, const float *D,
                  const void *lambda) {
    const size_t es = d->dtype_io == SSM_BF16 ? 2 : 4;
    int rc;
    if ((rc = check_ptr(x, "x", es)) || (rc = check_ptr(dt, "dt", es)) ||
        (rc = check_ptr(A_log, "A_log", 4)) || (rc = check_ptr(B, "B", es)) ||
        (rc = check_ptr(C, "C", es)))
        return rc;
    if (d->n_pairs > 0 && (rc = check_ptr(theta, "theta", 4))) return rc;
    if (d->rank_in == d->rank_out && (rc = check_ptr(D, "D", 4))) return rc;
    if (d->two_endpoint && (rc = check_ptr(lambda, "lambda", es))) return rc;
    return SSM_OK;
}

}  // namespace

namespace ssm {
void profile_mark(cudaStream_t st, const char *name) {
    if (!g_prof.active || g_prof.cur < 0 || g_prof.used >= g_prof.pool.size()) return;
    cudaEventRecord(g_prof.pool[g_prof.used], st);
    g_prof.recs.push_back({name, g_prof.cur, (int)g_prof.used});
    g_prof.cur = (int)g_prof.used++;
}
}  // namespace ssm

extern "C" {

void ssm_desc_set_contiguous(ssm_desc_t *d) {
    if (!d) return;
    const int64_t N = d->n_real + 2LL * d->n_pairs;
    const int64_t H = d->nheads, G = d->ngroups, L = d->seqlen, P = d->headdim;
    const int64_t R = d->rank_in, O = d->rank_out;
    d->stride_x[2] = R * P;
    d->stride_x[1] = H * R * P;
    d->stride_x[0] = L * H * R * P;
    d->stride_y[2] = O * P;
    d->stride_y[1] = H * O * P;
    d->stride_y[0] = L * H * O * P;
    d->stride_B[2] = R * N;
    d->stride_B[1] = G * R * N;
    d->stride_B[0] = L * G * R * N;
    d->stride_C[2] = O * N;
    d->stride_C[1] = G * O * N;
    d->stride_C[0] = L * G * O * N;
    d->stride_dt[2] = 1;
    d->stride_dt[1] = H;
    d->stride_dt[0] = L * H;
    for (int k = 0; k < 3; ++k) d->stride_lambda[k] = d->stride_dt[k];
}

size_t ssm_scan_workspace_size(const ssm_desc_t *d, int pass) {
    if (validate_desc(d) != SSM_OK) return 0;
    if (pass == SSM_PASS_FWD) return (d->batch == 0 || d->seqlen == 0) ? 0 : fwd_layout(d).total;
    if (pass == SSM_PASS_FWD_INFER)
        return (d->batch == 0 || d->seqlen == 0) ? 0 : fwd_layout(d).total_infer;
    if (pass != SSM_PASS_BWD) return 0;
    if (d->batch == 0 || d->seqlen == 0) return 0;
    // the chain the call takes with 16-byte aligned tensors
    if (m1_shape(d) && m1_strides(d)) return m1_bwd_bytes(d);
    if (ssd_shape(d) && ssd_strides(d)) return ssd_bwd_layout(d).total;
    return bwd_layout(d).total;
}

int ssm_preact_fwd(const ssm_desc_t *d, const void *z, const float *dt_bias,
                   const void *lambda_logit, void *dt, void *lambda, void *stream) {
    int rc = validate_desc(d);
    if (rc) return rc;
    if (d->batch == 0 || d->seqlen == 0) return SSM_OK;
    const size_t es = d->dtype_io == SSM_BF16 ? 2 : 4;
    if ((rc = check_ptr(z, "z", es)) || (rc = check_ptr(dt_bias, "dt_bias", 4)) ||
        (rc = check_ptr(dt, "dt", es)))
        return rc;
    if (d->two_endpoint && ((rc = check_ptr(lambda_logit, "lambda_logit", es)) ||
                            (rc = check_ptr(lambda, "lambda", es))))
        return rc;
    ssm::Params p;
    fill_params(d, p);
    ssm::PreactArgs a = {};
    a.z = z; a.bias = dt_bias; a.lam_logit = lambda_logit; a.dt = dt; a.lam = lambda;
    cudaStream_t st = (cudaStream_t)stream;
    profile_begin(st);
    const cudaError_t e = ssm::preact_forward(p, a, st);
    profile_end();
    if (e != cudaSuccess) return cuda_fail(e, "ssm_preact_fwd launch");
    g_last_error.clear();
    return SSM_OK;
}

int ssm_preact_bwd(const ssm_desc_t *d, const void *z, const float *dt_bias,
                   const void *lambda_logit, const void *ddt, const void *dlambda, void *dz,
                   float *ddt_bias, void *dlambda_logit, void *stream) {
    int rc = validate_desc(d);
    if (rc) return rc;
    cudaStream_t st = (cudaStream_t)stream;
    if (d->batch == 0 || d->seqlen == 0) {
        if (ddt_bias) {
            const cudaError_t e = cudaMemsetAsync(ddt_bias, 0, sizeof(float) * d->nheads, st);
            if (e != cudaSuccess) return cuda_fail(e, "ssm_preact_bwd (empty)");
        }
        return SSM_OK;
    }
    const size_t es = d->dtype_io == SSM_BF16 ? 2 : 4;
    if ((rc = check_ptr(z, "z", es)) || (rc = check_ptr(dt_bias, "dt_bias", 4)) ||
        (rc = check_ptr(ddt, "ddt", es)) || (rc = check_ptr(dz, "dz", es)))
        return rc;
    if (ddt_bias && (uintptr_t)ddt_bias % 4) return fail(SSM_ERR_ALIGN, "ddt_bias is not 4-byte aligned");
    if (d->two_endpoint && ((rc = check_ptr(lambda_logit, "lambda_logit", es)) ||
                            (rc = check_ptr(dlambda, "dlambda", es)) ||
                            (rc = check_ptr(dlambda_logit, "dlambda_logit", es))))
        return rc;
    ssm::Params p;
    fill_params(d, p);
    ssm::PreactArgs a = {};
    a.z = z; a.bias = dt_bias; a.lam_logit = lambda_logit; a.ddt = ddt; a.dlam = dlambda;
    a.dz = dz; a.dbias = ddt_bias; a.dlam_logit = dlambda_logit;
    profile_begin(st);
    const cudaError_t e = ssm::preact_backward(p, a, st);
    profile_end();
    if (e != cudaSuccess) return cuda_fail(e, "ssm_preact_bwd launch");
    g_last_error.clear();
    return SSM_OK;
}

int ssm_scan_step(const ssm_desc_t *d, const void *x, const void *dt, const float *A_log,
                  const float *theta, const void *B, const void *C, const float *D,
                  const void *lambda, float *h, float *w, void *y, void *stream) {
    int rc = validate_desc(d);
    if (rc) return rc;
    if (d->seqlen != 1) return fail(SSM_ERR_ARG, "ssm_scan_step takes one token (seqlen %lld)",
                                    (long long)d->seqlen);
    if (d->batch == 0) return SSM_OK;
    if ((rc = common_inputs(d, x, dt, A_log, theta, B, C, D, lambda))) return rc;
    if ((rc = check_ptr(y, "y", d->dtype_io == SSM_BF16 ? 2 : 4))) return rc;
    if ((rc = check_ptr(h, "h", 4))) return rc;
    if (d->two_endpoint && (rc = check_ptr(w, "w", 4))) return rc;
    if (w && (uintptr_t)w % 4) return fail(SSM_ERR_ALIGN, "w is not 4-byte aligned");
    ssm::Params p;
    fill_params(d, p);
    if (!ssm::step_supported(p))
        return fail(SSM_ERR_UNSUPPORTED, "ssm_scan_step: rank_in %d / rank_out %d above 8",
                    d->rank_in, d->rank_out);
    p.x = x; p.dt = dt; p.A_log = A_log; p.theta = theta; p.Bm = B; p.Cm = C; p.D = D;
    p.lam = lambda; p.y = y;
    cudaStream_t st = (cudaStream_t)stream;
    profile_begin(st);
    const cudaError_t e = ssm::scan_step(p, h, w, st);
    profile_end();
    if (e != cudaSuccess) return cuda_fail(e, "ssm_scan_step launch");
    g_last_error.clear();
    return SSM_OK;
}

}  // extern "C"

namespace {
// Forward of both entry points; z (may be NULL: no gate) is the mixer's output gate,
// applied by one elementwise pass after the chain that ran; y_pre (may be NULL)
// keeps the pre-gate y.
int fwd_impl(const ssm_desc_t *d, const void *x, const void *dt, const float *A_log,
             const float *theta, const void *B, const void *C, const float *D,
             const void *lambda, const float *h0, const float *prev_write, const void *z,
             void *y, void *y_pre, float *hT, float *last_write, void *workspace,
             size_t workspace_bytes, void *stream) {
    int rc = validate_desc(d);
    if (rc) return rc;
    if (d->batch == 0) return SSM_OK;
    if (d->seqlen > 0) {
        if ((rc = common_inputs(d, x, dt, A_log, theta, B, C, D, lambda))) return rc;
        const size_t es = d->dtype_io == SSM_BF16 ? 2 : 4;
        // y may be NULL for a state-only forward (hT / last_write), not with a gate
        if (y || z) {
            if ((rc = check_ptr(y, "y", es))) return rc;
        } else if (!hT && !last_write) {
            return fail(SSM_ERR_ARG, "y, hT and last_write are all NULL");
        }
        if (z && (uintptr_t)z % es) return fail(SSM_ERR_ALIGN, "z is not %zu-byte aligned", es);
        if (y_pre && (uintptr_t)y_pre % es)
            return fail(SSM_ERR_ALIGN, "y_pre is not %zu-byte aligned", es);
    }
    ssm::Params p;
    fill_params(d, p);
    p.x = x; p.dt = dt; p.A_log = A_log; p.theta = theta; p.Bm = B; p.Cm = C; p.D = D;
    p.lam = lambda; p.h0 = h0; p.w0 = prev_write; p.y = y; p.hT = hT; p.wT = last_write;
    p.gz = d->seqlen > 0 ? z : nullptr;
    p.ypre = p.gz ? y_pre : nullptr;
    // chunk == 1 asks for the token-by-token recurrent kernels
    if (m1_shape(d) && ssm::m1_supported(p)) {
        const FwdWs lay = fwd_layout(d);
        float *kept = nullptr;
        if (workspace && workspace_bytes >= lay.total) {
            if ((uintptr_t)workspace % 256) return fail(SSM_ERR_ALIGN, "workspace is not 256-byte aligned");
            kept = (float *)workspace;
        }
        cudaStream_t st = (cudaStream_t)stream;
        profile_begin(st);
        cudaError_t e = ssm::m1_forward(p, kept, st);
        if (e == cudaSuccess && p.gz) e = ssm::gate_forward(p, st);
        profile_end();
        g_last_gate = nullptr;
        g_last_route = SSM_ROUTE_CHANNEL;
        if (e != cudaSuccess) return cuda_fail(e, "ssm_scan_fwd launch");
        g_last_error.clear();
        return SSM_OK;
    }
    const bool ssd = ssd_shape(d) && ssm::ssd_supported(p);
    const bool chunked =
        !ssd && d->chunk != 1 && ssm::chunk_fwd_supported(p) && tensor_chain_shape(d);
    if (!ssd && !chunked && !ssm::simt_supported(p))
        return fail(SSM_ERR_UNSUPPORTED, "no kernel for n_real=%d n_pairs=%d P=%lld R=%d O=%d",
                    d->n_real, d->n_pairs, (long long)d->headdim, d->rank_in, d->rank_out);
    cudaStream_t st = (cudaStream_t)stream;
    if (ssd) {
        const FwdWs lay = fwd_layout(d);
        if (!workspace || workspace_bytes < lay.total_infer)
            return fail(SSM_ERR_WORKSPACE,
                        "forward needs %zu bytes of workspace (%zu to save for the backward), got %zu",
                        lay.total_infer, lay.total, workspace ? workspace_bytes : (size_t)0);
        if ((uintptr_t)workspace % 256)
            return fail(SSM_ERR_ALIGN, "workspace is not 256-byte aligned");
        char *ws = (char *)workspace;
        p.ws_ring = (float *)(ws + lay.off_ring);
        p.ws_flag = (int *)(ws + lay.off_flag);
        if (workspace_bytes >= lay.total) p.ws_kp = (float *)(ws + lay.off_kp);
        const int qt = ssm::ssd_chunk_tokens(ssd_rank(d));
        p.nc = (int)((d->seqlen + qt - 1) / qt);
        profile_begin(st);
        cudaError_t e = ssm::ssd_forward(p, st);
        if (e == cudaSuccess && p.gz) e = ssm::gate_forward(p, st);
        profile_end();
        g_last_gate = nullptr;
        g_last_route = SSM_ROUTE_SSD;
        if (e != cudaSuccess) return cuda_fail(e, "ssm_scan_fwd launch");
        g_last_error.clear();
        return SSM_OK;
    }
    // state-only forward on the per-coordinate chain: every chunk's state at once and
    // the carry pass (the backward's state rebuild), into the training workspace
    const bool states_only = chunked && !y && d->seqlen > 0;
    if (chunked) {
        const FwdWs lay = fwd_layout(d);
        if (states_only && (!workspace || workspace_bytes < lay.total))
            return fail(SSM_ERR_WORKSPACE,
                        "a state-only forward needs %zu bytes of workspace, got %zu", lay.total,
                        workspace ? workspace_bytes : (size_t)0);
        if (!workspace || workspace_bytes < lay.total_infer)
            return fail(SSM_ERR_WORKSPACE,
                        "forward needs %zu bytes of workspace (%zu to save for the backward), got %zu",
                        lay.total_infer, lay.total, workspace ? workspace_bytes : (size_t)0);
        if ((uintptr_t)workspace % 256)
            return fail(SSM_ERR_ALIGN, "workspace is not 256-byte aligned");
        char *ws = (char *)workspace;
        p.ws_ring = (float *)(ws + lay.off_ring);
        p.ws_flag = (int *)(ws + lay.off_flag);
        if (workspace_bytes >= lay.total) {  // training forward: keep the states and products
            p.ws_kp = (float *)(ws + lay.off_kp);
            p.ws_ce = (float *)(ws + lay.off_ce);
            p.sv_P = (unsigned char *)(ws + lay.off_P);
            p.sv_Bh = (unsigned char *)(ws + lay.off_Bh);
            p.sv_corr = (float *)(ws + lay.off_corr);
        }
        p.nc = (int)((d->seqlen + 63) / 64);
    }
    profile_begin(st);
    cudaError_t e = cudaSuccess;
    if (chunked) {
        // both chains are launched; the range check picks one on the device
        int *gate = nullptr;
        const bool fallback = ssm::simt_supported(p);
        if (fallback) {
            e = gate_slot(&gate, st);
            if (e == cudaSuccess) e = ssm::chunk_range_check(p, gate, st);
        }
        ssm::Params pc = p;
        pc.gate = gate;
        pc.gate_on = 0;
        if (e == cudaSuccess) {
            if (states_only) {
                pc.sv_P = nullptr;   // nothing else of the training forward is kept
                pc.sv_Bh = nullptr;
                pc.sv_corr = nullptr;
                e = ssm::chunk_states(pc, st);
            } else {
                e = ssm::chunk_forward(pc, st);
            }
        }
        if (e == cudaSuccess && fallback) {
            ssm::Params ps = p;
            ps.gate = gate;
            ps.gate_on = 1;
            e = ssm::simt_forward(ps, st);
        }
        // whichever chain ran wrote y: one gate pass (it reads y while it is in L2)
        if (e == cudaSuccess && p.gz) e = ssm::gate_forward(p, st);
        g_last_gate = gate;
        g_last_route = SSM_ROUTE_CHUNKED;
    } else {
        e = ssm::simt_forward(p, st);
        if (e == cudaSuccess && p.gz) e = ssm::gate_forward(p, st);
        g_last_gate = nullptr;
        g_last_route = SSM_ROUTE_RECURRENT;
    }
    profile_end();
    if (e != cudaSuccess) return cuda_fail(e, "ssm_scan_fwd launch");
    g_last_error.clear();
    return SSM_OK;
}
}  // namespace

extern "C" {

int ssm_scan_fwd(const ssm_desc_t *d, const void *x, const void *dt, const float *A_log,
                 const float *theta, const void *B, const void *C, const float *D,
                 const void *lambda, const float *h0, const float *prev_write, void *y,
                 float *hT, float *last_write, void *workspace, size_t workspace_bytes,
                 void *stream) {
    return fwd_impl(d, x, dt, A_log, theta, B, C, D, lambda, h0, prev_write, nullptr, y, nullptr,
                    hT, last_write, workspace, workspace_bytes, stream);
}

int ssm_scan_fwd_gated(const ssm_desc_t *d, const void *x, const void *dt, const float *A_log,
                       const float *theta, const void *B, const void *C, const float *D,
                       const void *lambda, const float *h0, const float *prev_write,
                       const void *z, void *y_gated, void *y_pre, float *hT, float *last_write,
                       void *workspace, size_t workspace_bytes, void *stream) {
    if (d && d->batch > 0 && d->seqlen > 0) {
        const int rc = check_ptr(z, "z", d->dtype_io == SSM_BF16 ? 2 : 4);
        if (rc) return rc;
    }
    return fwd_impl(d, x, dt, A_log, theta, B, C, D, lambda, h0, prev_write, z, y_gated, y_pre,
                    hT, last_write, workspace, workspace_bytes, stream);
}

int ssm_gate_bwd(const ssm_desc_t *d, const void *z, const void *y_pre, const void *dy_gated,
                 void *dy, void *dz, void *stream) {
    int rc = validate_desc(d);
    if (rc) return rc;
    if (d->batch == 0 || d->seqlen == 0) return SSM_OK;
    const size_t es = d->dtype_io == SSM_BF16 ? 2 : 4;
    if ((rc = check_ptr(z, "z", es)) || (rc = check_ptr(y_pre, "y_pre", es)) ||
        (rc = check_ptr(dy_gated, "dy_gated", es)) || (rc = check_ptr(dy, "dy", es)) ||
        (rc = check_ptr(dz, "dz", es)))
        return rc;
    ssm::Params p;
    fill_params(d, p);
    p.gz = z;
    p.ypre = const_cast<void *>(y_pre);
    cudaStream_t st = (cudaStream_t)stream;
    profile_begin(st);
    const cudaError_t e = ssm::gate_backward(p, dy_gated, dy, dz, st);
    profile_end();
    if (e != cudaSuccess) return cuda_fail(e, "ssm_gate_bwd launch");
    g_last_error.clear();
    return SSM_OK;
}

namespace {
// Backward of both entry points; `saved` (may be NULL) is the workspace of a
// forward call with the same descriptor and inputs, whose chunk states are
// then read instead of recomputed.
int bwd_impl(const ssm_desc_t *d, const void *x, const void *dt, const float *A_log,
             const float *theta, const void *B, const void *C, const float *D, const void *lambda,
             const float *h0, const float *prev_write, const void *dy, void *dx, void *ddt,
             float *dA_log, float *dtheta, void *dB, void *dC, float *dD, void *dlambda,
             float *dh0, float *dprev_write, const void *saved, size_t saved_bytes,
             void *workspace, size_t workspace_bytes, void *stream) {
    int rc = validate_desc(d);
    if (rc) return rc;
    const size_t es = d->dtype_io == SSM_BF16 ? 2 : 4;
    if ((rc = check_ptr(dA_log, "dA_log", 4))) return rc;
    if (d->rank_in == d->rank_out && (rc = check_ptr(dD, "dD", 4))) return rc;
    cudaStream_t st = (cudaStream_t)stream;
    if (d->batch == 0) return SSM_OK;
    if (d->seqlen == 0) {
        // nothing flows back through an empty sequence: zero parameter and state grads
        cudaError_t e = cudaMemsetAsync(dA_log, 0, sizeof(float) * d->nheads * ndecay(d), st);
        if (e == cudaSuccess && dtheta && d->n_pairs && d->angle_mode == SSM_ANGLE_STATIC)
            e = cudaMemsetAsync(dtheta, 0, sizeof(float) * d->nheads * d->n_pairs, st);
        if (e == cudaSuccess && dD) e = cudaMemsetAsync(dD, 0, sizeof(float) * d->nheads, st);
        size_t sb = sizeof(float) * d->batch * d->nheads * nstate(d) * d->headdim;
        if (e == cudaSuccess && dh0) e = cudaMemsetAsync(dh0, 0, sb, st);
        if (e == cudaSuccess && dprev_write) e = cudaMemsetAsync(dprev_write, 0, sb, st);
        if (e != cudaSuccess) return cuda_fail(e, "ssm_scan_bwd (empty sequence)");
        return SSM_OK;
    }
    if ((rc = common_inputs(d, x, dt, A_log, theta, B, C, D, lambda))) return rc;
    if ((rc = check_ptr(dy, "dy", es)) || (rc = check_ptr(dx, "dx", es)) ||
        (rc = check_ptr(ddt, "ddt", es)) || (rc = check_ptr(dB, "dB", es)) ||
        (rc = check_ptr(dC, "dC", es)))
        return rc;
    if (d->n_pairs > 0 && (rc = check_ptr(dtheta, "dtheta", 4))) return rc;
    if (dlambda && ((uintptr_t)dlambda % es)) return fail(SSM_ERR_ALIGN, "dlambda misaligned");
    const BwdWs lay = bwd_layout(d);
    if (saved) {
        const size_t need = fwd_layout(d).total;
        if (need == 0) {
            saved = nullptr;  // the recurrent kernels save nothing
        } else if (saved_bytes < need) {
            return fail(SSM_ERR_WORKSPACE, "saved forward workspace needs %zu bytes, got %zu",
                        need, saved_bytes);
        } else if ((uintptr_t)saved % 256) {
            return fail(SSM_ERR_ALIGN, "saved forward workspace is not 256-byte aligned");
        }
    }
    ssm::Params p;
    fill_params(d, p);
    p.x = x; p.dt = dt; p.A_log = A_log; p.theta = theta; p.Bm = B; p.Cm = C; p.D = D;
    p.lam = lambda; p.h0 = h0; p.w0 = prev_write; p.dy = dy;
    p.dx = dx; p.ddt = ddt; p.dA_log = dA_log; p.dtheta = dtheta; p.dBm = dB; p.dCm = dC;
    p.dD = dD; p.dlam = d->two_endpoint ? dlambda : nullptr; p.dh0 = dh0; p.dw0 = dprev_write;
    char *ws = (char *)workspace;
    p.ws_dC = (float *)(ws + lay.off_dC);
    p.ws_gbu = (float *)(ws + lay.off_gbu);
    p.ws_tok = (float *)(ws + lay.off_tok);
    p.ws_M2 = (float *)(ws + lay.off_M2);
    p.ws_par = (float *)(ws + lay.off_par);
    p.ws_ddt = (float *)(ws + lay.off_ddt);
    p.ws_blk = (float *)(ws + lay.off_blk);
    p.ws_blkc = (float *)(ws + lay.off_blkc);
    p.nc = (int)((d->seqlen + 63) / 64);
    // the chain this call takes, and the workspace it needs
    const bool use_m1 = m1_shape(d) && ssm::m1_supported(p);
    const bool use_ssd = !use_m1 && ssd_shape(d) && ssm::ssd_supported(p) &&
                         ((uintptr_t)dy & 15) == 0 && ((uintptr_t)dx & 15) == 0 &&
                         (d->nheads != d->ngroups || ((((uintptr_t)dB | (uintptr_t)dC) & 15) == 0));
    const size_t need_ws = use_m1 ? m1_bwd_bytes(d) : use_ssd ? ssd_bwd_layout(d).total : lay.total;
    if (!workspace || workspace_bytes < need_ws)
        return fail(SSM_ERR_WORKSPACE,
                    "backward needs %zu bytes of workspace, got %zu%s", need_ws,
                    workspace ? workspace_bytes : (size_t)0,
                    need_ws > ssm_scan_workspace_size(d, SSM_PASS_BWD)
                        ? " (tensors that are not 16-byte aligned take the recurrent kernels, "
                          "which need more than ssm_scan_workspace_size reports)"
                        : "");
    if ((uintptr_t)workspace % 256) return fail(SSM_ERR_ALIGN, "workspace is not 256-byte aligned");
    if (use_m1) {
        const size_t kb = align256(ssm::m1_kept_floats(d->batch, d->seqlen, d->nheads, nstate(d)) * 4);
        float *kept = (float *)ws;
        bool ready = false;
        if (saved) {
            kept = (float *)saved;
            ready = true;
        }
        profile_begin(st);
        const cudaError_t e = ssm::m1_backward(p, kept, ready, (float *)(ws + kb), st);
        profile_end();
        g_last_gate = nullptr;
        g_last_route = SSM_ROUTE_CHANNEL;
        if (e != cudaSuccess) return cuda_fail(e, "ssm_scan_bwd launch");
        g_last_error.clear();
        return SSM_OK;
    }
    if (saved && m1_shape(d)) saved = nullptr;   // states kept by the channel scan: not read here
    if (use_ssd) {
        // scalar-decay chain
        const SsdBwdWs sl = ssd_bwd_layout(d);
        ssm::Params pc = p;
        pc.ws_ring = (float *)(ws + sl.off_ring);
        pc.ws_flag = (int *)(ws + sl.off_flag);
        pc.ws_kp = (float *)(ws + sl.off_kp);
        pc.sd_tok = (float *)(ws + sl.off_tok);
        pc.sd_par = (float *)(ws + sl.off_par);
        pc.sd_db0 = (float *)(ws + sl.off_db0);
        if (d->nheads != d->ngroups) {
            pc.sd_dBh = (float *)(ws + sl.off_dBh);
            pc.sd_dCh = (float *)(ws + sl.off_dCh);
        }
        const int qt = ssm::ssd_chunk_tokens(ssd_rank(d));
        pc.nc = (int)((d->seqlen + qt - 1) / qt);
        if (saved) {
            pc.ws_kp = (float *)((const char *)saved + fwd_layout(d).off_kp);
            pc.states_ready = 1;
        }
        profile_begin(st);
        const cudaError_t e = ssm::ssd_backward(pc, st);
        profile_end();
        g_last_gate = nullptr;
        g_last_route = SSM_ROUTE_SSD;
        if (e != cudaSuccess) return cuda_fail(e, "ssm_scan_bwd launch");
        g_last_error.clear();
        return SSM_OK;
    }
    if (saved && ssd_shape(d)) saved = nullptr;   // scalar-decay forward states: not read here
    if (!ssm::simt_supported(p))
        return fail(SSM_ERR_UNSUPPORTED, "no kernel for n_real=%d n_pairs=%d P=%lld R=%d O=%d",
                    d->n_real, d->n_pairs, (long long)d->headdim, d->rank_in, d->rank_out);
    // dD is written by the parameter pass; keep it defined when R != O
    const bool chunked = d->chunk != 1 && ssm::chunk_bwd_supported(p) && lay.boundary;
    profile_begin(st);
    cudaError_t e = cudaSuccess;
    if (chunked) {
        // both chains are launched; the range check picks one on the device
        int *gate = nullptr;
        e = gate_slot(&gate, st);
        if (e == cudaSuccess) e = ssm::chunk_range_check(p, gate, st);
        ssm::Params pc = p;
        pc.ws_kp = (float *)(ws + lay.off_kp);
        pc.ws_qb = (float *)(ws + lay.off_qb);
        pc.ws_gc = (float *)(ws + lay.off_gc);
        pc.ws_ce = (float *)(ws + lay.off_ce);
        pc.ws_ring = (float *)(ws + lay.off_ring);
        pc.ws_flag = (int *)(ws + lay.off_flag);
        if (saved) {
            // read-only here: the forward wrote them
            const FwdWs fl = fwd_layout(d);
            const char *sv = (const char *)saved;
            pc.ws_kp = (float *)(sv + fl.off_kp);
            pc.ws_ce = (float *)(sv + fl.off_ce);
            pc.sv_P = (unsigned char *)(sv + fl.off_P);
            pc.sv_Bh = (unsigned char *)(sv + fl.off_Bh);
            pc.sv_corr = (float *)(sv + fl.off_corr);
            pc.states_ready = 1;
        }
        pc.gate = gate;
        pc.gate_on = 0;
        if (e == cudaSuccess) e = ssm::chunk_backward(pc, st);
        ssm::Params ps = p;
        ps.gate = gate;
        ps.gate_on = 1;
        if (e == cudaSuccess) e = ssm::simt_backward(ps, st);
        g_last_gate = gate;
        g_last_route = SSM_ROUTE_CHUNKED;
    } else {
        e = ssm::simt_backward(p, st);
        g_last_gate = nullptr;
        g_last_route = SSM_ROUTE_RECURRENT;
    }
    profile_end();
    if (e != cudaSuccess) return cuda_fail(e, "ssm_scan_bwd launch");
    g_last_error.clear();
    return SSM_OK;
}

}  // namespace

int ssm_scan_bwd(const ssm_desc_t *d, const void *x, const void *dt, const float *A_log,
                 const float *theta, const void *B, const void *C, const float *D,
                 const void *lambda, const float *h0, const float *prev_write, const void *dy,
                 void *dx, void *ddt, float *dA_log, float *dtheta, void *dB, void *dC,
                 float *dD, void *dlambda, float *dh0, float *dprev_write, void *workspace,
                 size_t workspace_bytes, void *stream) {
    return bwd_impl(d, x, dt, A_log, theta, B, C, D, lambda, h0, prev_write, dy, dx, ddt, dA_log,
                    dtheta, dB, dC, dD, dlambda, dh0, dprev_write, nullptr, 0, workspace,
                    workspace_bytes, stream);
}

int ssm_scan_bwd_saved(const ssm_desc_t *d, const void *x, const void *dt, const float *A_log,
                       const float *theta, const void *B, const void *C, const float *D,
                       const void *lambda, const float *h0, const float *prev_write,
                       const void *dy, void *dx, void *ddt, float *dA_log, float *dtheta,
                       void *dB, void *dC, float *dD, void *dlambda, float *dh0,
                       float *dprev_write, const void *fwd_workspace,
                       size_t fwd_workspace_bytes, void *workspace, size_t workspace_bytes,
                       void *stream) {
    if (!fwd_workspace) return fail(SSM_ERR_ARG, "ssm_scan_bwd_saved: fwd_workspace is NULL");
    return bwd_impl(d, x, dt, A_log, theta, B, C, D, lambda, h0, prev_write, dy, dx, ddt, dA_log,
                    dtheta, dB, dC, dD, dlambda, dh0, dprev_write, fwd_workspace,
                    fwd_workspace_bytes, workspace, workspace_bytes, stream);
}

const char *ssm_scan_last_error(void) { return g_last_error.c_str(); }

int ssm_scan_poll_device_error(void *stream) {
    cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "ssm_scan_poll_device_error");
    int word = ssm::chunk_error_take();
    const int word2 = ssm::chunk_rev_error_take();
    if (word == 0 || word2 < 0) word = word2;
    const int word3 = ssm::ssd_error_take();
    if (word == 0 || word3 < 0) word = word3;
    if (word < 0) return fail(SSM_ERR_CUDA, "ssm_scan_poll_device_error: cannot read the error word");
    if (word == 1) return fail(SSM_ERR_TIMEOUT, "a bounded device-side wait gave up");
    if (word != 0) return fail(SSM_ERR_TIMEOUT, "device-side error code %d", word);
    return SSM_OK;
}

int ssm_scan_abi_version(void) { return SSM_SCAN_ABI_VERSION; }

int64_t ssm_scan_set_wait_limit(int64_t polls) {
    if (polls < 0) return fail(SSM_ERR_ARG, "wait limit must be >= 0");
    return (int64_t)g_wait_limit.exchange((long long)polls);
}

int ssm_scan_last_route(void *stream) {
    if (g_last_route < 0) return fail(SSM_ERR_ARG, "no scan call on this thread yet");
    if (g_last_route != SSM_ROUTE_CHUNKED || !g_last_gate) return g_last_route;
    cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "ssm_scan_last_route");
    int v = 0;
    e = cudaMemcpy(&v, g_last_gate, sizeof(int), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_fail(e, "ssm_scan_last_route (gate word)");
    return v ? SSM_ROUTE_RANGE_FALLBACK : SSM_ROUTE_CHUNKED;
}

int ssm_scan_profile_start(int max_launches) {
    if (max_launches < 1) return fail(SSM_ERR_ARG, "max_launches must be >= 1");
    if (g_prof.active) return fail(SSM_ERR_ARG, "a profiling session is already open");
    g_prof = ProfileSession();
    const size_t n = (size_t)max_launches + 64;
    g_prof.pool.resize(n);
    for (size_t i = 0; i < n; ++i) {
        cudaError_t e = cudaEventCreate(&g_prof.pool[i]);
        if (e != cudaSuccess) {
            for (size_t k = 0; k < i; ++k) cudaEventDestroy(g_prof.pool[k]);
            g_prof = ProfileSession();
            return cuda_fail(e, "ssm_scan_profile_start");
        }
    }
    g_prof.active = true;
    return SSM_OK;
}

int ssm_scan_profile_stop(char *names, int name_len, int *counts, double *total_ms,
                          int max_kernels) {
    if (!g_prof.active) return fail(SSM_ERR_ARG, "no profiling session is open");
    int rc = SSM_OK;
    std::vector<std::string> seen;
    std::vector<int> cnt;
    std::vector<double> tot;
    if (g_prof.used > 0) {
        cudaError_t e = cudaEventSynchronize(g_prof.pool[g_prof.used - 1]);
        if (e != cudaSuccess) rc = cuda_fail(e, "ssm_scan_profile_stop");
    }
    if (rc == SSM_OK) {
        for (const ProfileRec &r : g_prof.recs) {
            float ms = 0.f;
            cudaError_t e = cudaEventElapsedTime(&ms, g_prof.pool[r.ev0], g_prof.pool[r.ev1]);
            if (e != cudaSuccess) {
                rc = cuda_fail(e, "ssm_scan_profile_stop (elapsed)");
                break;
            }
            size_t k = 0;
            while (k < seen.size() && seen[k] != r.name) ++k;
            if (k == seen.size()) {
                seen.push_back(r.name);
                cnt.push_back(0);
                tot.push_back(0.0);
            }
            cnt[k] += 1;
            tot[k] += ms;
        }
    }
    for (cudaEvent_t ev : g_prof.pool) cudaEventDestroy(ev);
    g_prof = ProfileSession();
    if (rc != SSM_OK) return rc;
    int n = (int)seen.size() < max_kernels ? (int)seen.size() : max_kernels;
    for (int i = 0; i < n; ++i) {
        if (names && name_len > 0) {
            strncpy(names + (size_t)i * name_len, seen[i].c_str(), name_len - 1);
            names[(size_t)i * name_len + name_len - 1] = 0;
        }
        if (counts) counts[i] = cnt[i];
        if (total_ms) total_ms[i] = tot[i];
    }
    return n;
}


// ---- sequence sharding ---------------------------------------------------------------
int ssm_cp_tail_rows(const ssm_desc_t *d) {
    if (validate_desc(d)) return -1;
    return (d->dtype_io == SSM_BF16 ? 2 : 1) * nstate(d);
}

int ssm_cp_segment_transition(const ssm_desc_t *d, const void *dt, const float *A_log,
                              const float *theta, const void *lambda, float *phi, float *beta0,
                              void *stream) {
    int rc = validate_desc(d);
    if (rc) return rc;
    const size_t es = d->dtype_io == SSM_BF16 ? 2 : 4;
    if ((rc = check_ptr(dt, "dt", es)) || (rc = check_ptr(A_log, "A_log", 4)) ||
        (rc = check_ptr(phi, "phi", 4)) || (rc = check_ptr(beta0, "beta0", 4)))
        return rc;
    if (d->n_pairs && (rc = check_ptr(theta, "theta", 4))) return rc;
    if (d->two_endpoint && (rc = check_ptr(lambda, "lambda", es))) return rc;
    if (d->n_pairs > 64)
        return fail(SSM_ERR_UNSUPPORTED, "ssm_cp_segment_transition: n_pairs %d above 64", d->n_pairs);
    ssm::Params p;
    fill_params(d, p);
    p.dt = dt; p.A_log = A_log; p.theta = theta; p.lam = lambda;
    cudaStream_t st = (cudaStream_t)stream;
    profile_begin(st);
    const cudaError_t e = ssm::cp_transition(p, phi, beta0, st);
    profile_end();
    if (e != cudaSuccess) return cuda_fail(e, "ssm_cp_segment_transition launch");
    g_last_error.clear();
    return SSM_OK;
}

int ssm_cp_state_combine(const ssm_desc_t *d, int nseg, int seg, const float *hT_all,
                         const float *wT_all, const float *phi_all, const float *beta0_all,
                         const float *h0, const float *w0, float *h_in, float *w_in,
                         void *stream) {
    int rc = validate_desc(d);
    if (rc) return rc;
    if (nseg < 1 || seg < 0 || seg >= nseg)
        return fail(SSM_ERR_ARG, "ssm_cp_state_combine: segment %d of %d", seg, nseg);
    if ((rc = check_ptr(h_in, "h_in", 4)) || (rc = check_ptr(w_in, "w_in", 4))) return rc;
    if (seg > 0 && ((rc = check_ptr(hT_all, "hT_all", 4)) || (rc = check_ptr(wT_all, "wT_all", 4)) ||
                    (rc = check_ptr(phi_all, "phi_all", 4)) ||
                    (rc = check_ptr(beta0_all, "beta0_all", 4))))
        return rc;
    ssm::Params p;
    fill_params(d, p);
    cudaStream_t st = (cudaStream_t)stream;
    profile_begin(st);
    const cudaError_t e =
        ssm::cp_state_combine(p, seg, hT_all, wT_all, phi_all, beta0_all, h0, w0, h_in, w_in, st);
    profile_end();
    if (e != cudaSuccess) return cuda_fail(e, "ssm_cp_state_combine launch");
    g_last_error.clear();
    return SSM_OK;
}

int ssm_cp_adjoint_combine(const ssm_desc_t *d, int nseg, int seg, const float *dh0_all,
                           const float *phi_all, const float *beta0_all, const float *dhT,
                           float *dh_end, float *dw_end, void *stream) {
    int rc = validate_desc(d);
    if (rc) return rc;
    if (nseg < 1 || seg < 0 || seg >= nseg)
        return fail(SSM_ERR_ARG, "ssm_cp_adjoint_combine: segment %d of %d", seg, nseg);
    if ((rc = check_ptr(dh_end, "dh_end", 4)) || (rc = check_ptr(dw_end, "dw_end", 4))) return rc;
    if (seg + 1 < nseg &&
        ((rc = check_ptr(dh0_all, "dh0_all", 4)) || (rc = check_ptr(phi_all, "phi_all", 4)) ||
         (rc = check_ptr(beta0_all, "beta0_all", 4))))
        return rc;
    ssm::Params p;
    fill_params(d, p);
    cudaStream_t st = (cudaStream_t)stream;
    profile_begin(st);
    const cudaError_t e = ssm::cp_adjoint_combine(p, nseg, seg, dh0_all, phi_all, beta0_all, dhT,
                                                  dh_end, dw_end, st);
    profile_end();
    if (e != cudaSuccess) return cuda_fail(e, "ssm_cp_adjoint_combine launch");
    g_last_error.clear();
    return SSM_OK;
}

int ssm_cp_fill_tail(const ssm_desc_t *d, void *x, void *dt, void *B, void *C, void *lambda,
                     void *dy, const float *dh_end, void *stream) {
    int rc = validate_desc(d);
    if (rc) return rc;
    if (d->angle_mode == SSM_ANGLE_PER_TOKEN && d->n_pairs)
        return fail(SSM_ERR_UNSUPPORTED, "ssm_cp_fill_tail: per-token angles");
    if (d->n_static)
        return fail(SSM_ERR_UNSUPPORTED,
                    "ssm_cp_fill_tail: static rows (their transition does not vanish with dt)");
    const size_t es = d->dtype_io == SSM_BF16 ? 2 : 4;
    // x, dt, B, C and lambda all NULL: only the dy rows (the rest as an earlier call left them)
    const bool dy_only = !x && !dt && !B && !C && !lambda;
    if ((rc = check_ptr(dy, "dy", es))) return rc;
    if (!dy_only) {
        if ((rc = check_ptr(x, "x", es)) || (rc = check_ptr(dt, "dt", es)) ||
            (rc = check_ptr(B, "B", es)) || (rc = check_ptr(C, "C", es)))
            return rc;
        if (d->two_endpoint && (rc = check_ptr(lambda, "lambda", es))) return rc;
    }
    ssm::Params p;
    fill_params(d, p);
    p.x = x; p.dt = dt; p.Bm = B; p.Cm = C; p.lam = lambda; p.dy = dy;
    cudaStream_t st = (cudaStream_t)stream;
    profile_begin(st);
    const cudaError_t e = ssm::cp_fill_tail(p, ssm_cp_tail_rows(d), dh_end, st);
    profile_end();
    if (e != cudaSuccess) return cuda_fail(e, "ssm_cp_fill_tail launch");
    g_last_error.clear();
    return SSM_OK;
}

int ssm_cp_write_adjoint(const ssm_desc_t *d, const void *x, const void *B, const float *dw_end,
                         void *dx, void *dB, void *stream) {
    int rc = validate_desc(d);
    if (rc) return rc;
    if (d->batch == 0 || d->seqlen == 0) return SSM_OK;
    const size_t es = d->dtype_io == SSM_BF16 ? 2 : 4;
    if ((rc = check_ptr(x, "x", es)) || (rc = check_ptr(B, "B", es)) ||
        (rc = check_ptr(dw_end, "dw_end", 4)) || (rc = check_ptr(dx, "dx", es)) ||
        (rc = check_ptr(dB, "dB", es)))
        return rc;
    ssm::Params p;
    fill_params(d, p);
    p.x = x; p.Bm = B; p.dx = dx; p.dBm = dB;
    cudaStream_t st = (cudaStream_t)stream;
    profile_begin(st);
    const cudaError_t e = ssm::cp_write_adjoint(p, dw_end, st);
    profile_end();
    if (e != cudaSuccess) return cuda_fail(e, "ssm_cp_write_adjoint launch");
    g_last_error.clear();
    return SSM_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Allocation-free backward: the scratch lives in this fixed device array.
// Host code only ever sees the array's host-side shadow symbol, so its device
// address is looked up once per device (with that device current) and passed
// to the kernels as an ordinary pointer.
// ---------------------------------------------------------------------------
static __device__ __align__(256) unsigned char g_noalloc_scratch[SSM_NOALLOC_SCRATCH_BYTES];

namespace {
constexpr int kMaxDevices = 128;
std::mutex g_noalloc_mu;
void *g_noalloc_ptr[kMaxDevices];

int noalloc_scratch(void **out) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "ssm_scan_bwd_noalloc (cudaGetDevice)");
    if (dev < 0 || dev >= kMaxDevices) return fail(SSM_ERR_UNSUPPORTED, "device ordinal %d", dev);
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (!g_noalloc_ptr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess || !p)
            return cuda_fail(e, "ssm_scan_bwd_noalloc (cudaGetSymbolAddress)");
        g_noalloc_ptr[dev] = p;
    }
    *out = g_noalloc_ptr[dev];
    return SSM_OK;
}
}  // namespace

extern "C" int ssm_scan_bwd_noalloc(const ssm_desc_t *d, const void *x, const void *dt,
                                    const float *A_log, const float *theta, const void *B,
                                    const void *C, const float *D, const void *lambda,
                                    const float *h0, const float *prev_write, const void *dy,
                                    void *dx, void *ddt, float *dA_log, float *dtheta, void *dB,
                                    void *dC, float *dD, void *dlambda, float *dh0,
                                    float *dprev_write, void *stream) {
    int rc = validate_desc(d);
    if (rc) return rc;
    const size_t need = ssm_scan_workspace_size(d, SSM_PASS_BWD);
    if (need > (size_t)SSM_NOALLOC_SCRATCH_BYTES)
        return fail(SSM_ERR_WORKSPACE,
                    "ssm_scan_bwd_noalloc: this problem needs %zu bytes of scratch; the built-in "
                    "scratch holds %u bytes (use ssm_scan_bwd with a caller workspace)",
                    need, (unsigned)SSM_NOALLOC_SCRATCH_BYTES);
    void *scratch = nullptr;
    if ((rc = noalloc_scratch(&scratch))) return rc;
    return ssm_scan_bwd(d, x, dt, A_log, theta, B, C, D, lambda, h0, prev_write, dy, dx, ddt,
                        dA_log, dtheta, dB, dC, dD, dlambda, dh0, dprev_write, scratch,
                        SSM_NOALLOC_SCRATCH_BYTES, stream);
}
