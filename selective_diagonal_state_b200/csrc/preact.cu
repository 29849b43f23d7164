// Pre-activations of the step size and of the two-endpoint weight, and their
// gradients.  The step dt of a selective SSM is learned or input-dependent and
// is initialised log-uniform ("State Space Models", robocikowo.com: the
// entries on the discretisation step and its initialisation range).  Its
// positivity map and that of the two-endpoint weight are not spelled out on
// the pages; the reading taken here is the one the synthetic workloads use:
//     dt = softplus(z + dt_bias[h]),   lambda = sigmoid(lambda_logit)
// with dt_bias = log(expm1(dt0)) placing dt at dt0 for z = 0.
// Backward: dz = ddt * sigmoid(z + dt_bias), ddt_bias[h] = sum over (b, t) of
// dz, dlambda_logit = dlambda * lambda * (1 - lambda).
// One pass over [B][L][H] each way, every element its own thread.  The bias
// gradient is the per-head sum of the dz the backward returns: one cluster of
// eight CTAs per group of 32 heads (a lane per head, so a warp reads 32
// neighbouring heads of one (b, t) row at once) sums it, each CTA over its rows,
// and the cluster's first CTA adds the eight partial sums through distributed
// shared memory in CTA order: a fixed summation order (deterministic) with no
// workspace.
#include <cooperative_groups.h>

#include <initializer_list>

#include "common.cuh"

namespace ssm {

// argument block of the pre-activation kernels (declared alike in abi.cu)
struct PreactArgs {
    const void *z, *lam_logit, *ddt, *dlam;
    const float *bias;
    void *dt, *lam, *dz, *dlam_logit;
    float *dbias;
};

__device__ __forceinline__ float softplus_f(float x) {
    return x > 20.f ? x : log1pf(expf(x));
}
__device__ __forceinline__ float sigmoid_f(float x) { return __frcp_rn(1.f + __expf(-x)); }

// (b, t, h) of flat element i of [B][L][H] (32-bit divisions when the problem fits:
// the 64-bit ones are far slower)
__device__ __forceinline__ void preact_index(const Params &p, long long i, long long total, int &b,
                                             int &t, int &h) {
    if (total <= 0x7fffffffLL) {
        const unsigned iu = (unsigned)i, bt = iu / (unsigned)p.H;
        h = (int)(iu - bt * (unsigned)p.H);
        b = (int)(bt / (unsigned)p.L);
        t = (int)(bt - (unsigned)b * (unsigned)p.L);
    } else {
        h = (int)(i % p.H);
        const long long bt = i / p.H;
        t = (int)(bt % p.L);
        b = (int)(bt / p.L);
    }
}

// Elementwise passes.  With dense [B][L][H] layouts and an even head count
// (`pairs`), a thread takes two neighbouring heads of one (b, t) row with one
// 4- or 8-byte access per tensor and one division for the head index; otherwise
// one element with its (b, t, h) from the strides.
__device__ __forceinline__ float2 ld_io2(const void *ptr, long long i, int bf16) {
    if (bf16) {
        const uint32_t w = *reinterpret_cast<const uint32_t *>(reinterpret_cast<const __nv_bfloat16 *>(ptr) + i);
        return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
    }
    return *reinterpret_cast<const float2 *>(reinterpret_cast<const float *>(ptr) + i);
}
__device__ __forceinline__ void st_io2(void *ptr, long long i, float a, float b, int bf16) {
    if (bf16) {
        const __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
        *reinterpret_cast<__nv_bfloat162 *>(reinterpret_cast<__nv_bfloat16 *>(ptr) + i) = v;
    } else {
        *reinterpret_cast<float2 *>(reinterpret_cast<float *>(ptr) + i) = make_float2(a, b);
    }
}

__global__ void __launch_bounds__(256) k_preact_fwd(Params p, PreactArgs a, int pairs) {
    const long long total = (long long)p.Bsz * p.L * p.H;
    const long long stride = (long long)gridDim.x * blockDim.x;
    const bool lam = p.two_ep && a.lam;
    if (pairs) {
        for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; 2 * e < total;
             e += stride) {
            const long long i = 2 * e;
            const int h = (int)(total <= 0x7fffffffLL ? (unsigned)i % (unsigned)p.H : i % p.H);
            const float2 z = ld_io2(a.z, i, p.bf16);
            float2 lg = make_float2(0.f, 0.f);
            if (lam) lg = ld_io2(a.lam_logit, i, p.bf16);
            st_io2(a.dt, i, softplus_f(z.x + a.bias[h]), softplus_f(z.y + a.bias[h + 1]), p.bf16);
            if (lam) st_io2(a.lam, i, sigmoid_f(lg.x), sigmoid_f(lg.y), p.bf16);
        }
        return;
    }
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total; i += stride) {
        int b, t, h;
        preact_index(p, i, total, b, t, h);
        const long long id = ix_dt(p, b, t, h);
        st_io(a.dt, id, softplus_f(ld_io(a.z, id, p.bf16) + a.bias[h]), p.bf16);
        if (lam) {
            const long long il = ix_lam(p, b, t, h);
            st_io(a.lam, il, sigmoid_f(ld_io(a.lam_logit, il, p.bf16)), p.bf16);
        }
    }
}

// dz and dlambda_logit, elementwise
__global__ void __launch_bounds__(256) k_preact_bwd(Params p, PreactArgs a, int pairs) {
    const long long total = (long long)p.Bsz * p.L * p.H;
    const long long stride = (long long)gridDim.x * blockDim.x;
    const bool lam = p.two_ep && a.dlam_logit;
    if (pairs) {
        for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; 2 * e < total;
             e += stride) {
            const long long i = 2 * e;
            const int h = (int)(total <= 0x7fffffffLL ? (unsigned)i % (unsigned)p.H : i % p.H);
            const float2 z = ld_io2(a.z, i, p.bf16), g = ld_io2(a.ddt, i, p.bf16);
            float2 lg = make_float2(0.f, 0.f), dl = make_float2(0.f, 0.f);
            if (lam) {
                lg = ld_io2(a.lam_logit, i, p.bf16);
                dl = ld_io2(a.dlam, i, p.bf16);
            }
            st_io2(a.dz, i, g.x * sigmoid_f(z.x + a.bias[h]), g.y * sigmoid_f(z.y + a.bias[h + 1]),
                   p.bf16);
            if (lam) {
                const float s0 = sigmoid_f(lg.x), s1 = sigmoid_f(lg.y);
                st_io2(a.dlam_logit, i, dl.x * s0 * (1.f - s0), dl.y * s1 * (1.f - s1), p.bf16);
            }
        }
        return;
    }
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total; i += stride) {
        int b, t, h;
        preact_index(p, i, total, b, t, h);
        const long long id = ix_dt(p, b, t, h);
        st_io(a.dz, id, ld_io(a.ddt, id, p.bf16) * sigmoid_f(ld_io(a.z, id, p.bf16) + a.bias[h]),
              p.bf16);
        if (lam) {
            const long long il = ix_lam(p, b, t, h);
            const float sg = sigmoid_f(ld_io(a.lam_logit, il, p.bf16));
            st_io(a.dlam_logit, il, ld_io(a.dlam, il, p.bf16) * sg * (1.f - sg), p.bf16);
        }
    }
}

constexpr int PRE_CLUSTER = 16;   // CTAs per group of 32 heads (a non-portable cluster size)

// ddt_bias[h] = sum over (b, t) of dz[b][t][h] as written by k_preact_bwd
__global__ void __cluster_dims__(PRE_CLUSTER, 1, 1) __launch_bounds__(1024)
    k_preact_dbias(Params p, PreactArgs a) {
    namespace cg = cooperative_groups;
    __shared__ float part[32][33];   // [warp][lane]
    __shared__ float tot[32];        // this CTA's sum per head of the group
    cg::cluster_group cl = cg::this_cluster();
    const int rank = (int)cl.block_rank();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int h = (int)(blockIdx.x / PRE_CLUSTER) * 32 + lane;
    const bool hv = h < p.H;
    float acc = 0.f;
    if (hv) {
        // rows rank * 32 + warp + k * 32 * PRE_CLUSTER in (b, t) order, stepped without
        // divisions, sixteen loads in flight at a time
        constexpr int STRIDE = 32 * PRE_CLUSTER, U = 16;
        int b = 0, t = rank * 32 + warp;
        while (t >= p.L && b < p.Bsz) {
            t -= p.L;
            ++b;
        }
        while (b < p.Bsz) {
            float v[U];
#pragma unroll
            for (int k = 0; k < U; ++k) {
                v[k] = b < p.Bsz ? ld_io(a.dz, ix_dt(p, b, t, h), p.bf16) : 0.f;
                t += STRIDE;
                while (t >= p.L && b < p.Bsz) {
                    t -= p.L;
                    ++b;
                }
            }
#pragma unroll
            for (int k = 0; k < U; ++k) acc += v[k];
        }
    }
    part[warp][lane] = acc;
    __syncthreads();
    if (warp == 0) {
        float s = 0.f;
        for (int k = 0; k < 32; ++k) s += part[k][lane];
        tot[lane] = s;
    }
    cl.sync();   // every CTA's tot is written
    if (rank == 0 && warp == 0 && hv) {
        float s = 0.f;
        for (int k = 0; k < PRE_CLUSTER; ++k) s += cl.map_shared_rank(tot, k)[lane];
        a.dbias[h] = s;
    }
    cl.sync();   // no CTA leaves while the first one reads its shared memory
}

// Two neighbouring heads per thread when every tensor of the pass is dense
// [B][L][H] (strides L H, H, 1), the head count even and the pointers 8-byte aligned.
static int preact_pairs(const Params &p, std::initializer_list<const void *> ptrs) {
    if (p.H % 2) return 0;
    const long long LH = (long long)p.L * p.H;
    if (p.sdt[0] != LH || p.sdt[1] != p.H || p.sdt[2] != 1) return 0;
    if (p.two_ep && (p.slam[0] != LH || p.slam[1] != p.H || p.slam[2] != 1)) return 0;
    const uintptr_t al = p.bf16 ? 4 : 8;
    for (const void *q : ptrs)
        if (q && ((uintptr_t)q % al)) return 0;
    return 1;
}

// Blocks of the elementwise passes: at most sixteen blocks of 256 per SM (148
// SMs), looping past that.
static int preact_blocks(const Params &p, int pairs) {
    const long long total = (long long)p.Bsz * p.L * p.H;
    const long long per = pairs ? 512 : 256;
    long long blocks = (total + per - 1) / per;
    if (blocks > 148 * 16) blocks = 148 * 16;
    return blocks < 1 ? 1 : (int)blocks;
}

cudaError_t preact_forward(const Params &p, const PreactArgs &a, cudaStream_t st) {
    const int pairs = preact_pairs(p, {a.z, a.lam_logit, a.dt, a.lam});
    k_preact_fwd<<<preact_blocks(p, pairs), 256, 0, st>>>(p, a, pairs);
    profile_mark(st, "k_preact_fwd");
    return cudaGetLastError();
}

cudaError_t preact_backward(const Params &p, const PreactArgs &a, cudaStream_t st) {
    const int pairs = preact_pairs(p, {a.z, a.ddt, a.dz, a.lam_logit, a.dlam, a.dlam_logit});
    k_preact_bwd<<<preact_blocks(p, pairs), 256, 0, st>>>(p, a, pairs);
    profile_mark(st, "k_preact_bwd");
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess || !a.dbias) return e;
    static bool done[64] = {};   // the cluster size opt-in, per device
    int dev = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if (!(dev >= 0 && dev < 64 && done[dev])) {
        e = cudaFuncSetAttribute(k_preact_dbias, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        if (e != cudaSuccess) return e;
        if (dev >= 0 && dev < 64) done[dev] = true;
    }
    const int groups = (p.H + 31) / 32;
    k_preact_dbias<<<groups * PRE_CLUSTER, 1024, 0, st>>>(p, a);
    profile_mark(st, "k_preact_dbias");
    return cudaGetLastError();
}

}  // namespace ssm
