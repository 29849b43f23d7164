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
// One pass over [B][L][H] each way; the bias gradient is summed per head by
// one CTA in a fixed order (deterministic).
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
__device__ __forceinline__ float sigmoid_f(float x) { return 1.f / (1.f + expf(-x)); }

__global__ void __launch_bounds__(256) k_preact_fwd(Params p, PreactArgs a) {
    const long long total = (long long)p.Bsz * p.L * p.H;
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
         i += (long long)gridDim.x * blockDim.x) {
        const int h = (int)(i % p.H);
        const long long bt = i / p.H;
        const int t = (int)(bt % p.L), b = (int)(bt / p.L);
        const long long id = ix_dt(p, b, t, h);
        st_io(a.dt, id, softplus_f(ld_io(a.z, id, p.bf16) + a.bias[h]), p.bf16);
        if (p.two_ep && a.lam) {
            const long long il = ix_lam(p, b, t, h);
            st_io(a.lam, il, sigmoid_f(ld_io(a.lam_logit, il, p.bf16)), p.bf16);
        }
    }
}

// one CTA per head: every (b, t) of the head, then the fixed-order tree sum of dz
__global__ void __launch_bounds__(256) k_preact_bwd(Params p, PreactArgs a) {
    __shared__ float red[256];
    const int h = blockIdx.x, tid = threadIdx.x;
    const long long n = (long long)p.Bsz * p.L;
    float acc = 0.f;
    for (long long i = tid; i < n; i += blockDim.x) {
        const int t = (int)(i % p.L), b = (int)(i / p.L);
        const long long id = ix_dt(p, b, t, h);
        const float dz = ld_io(a.ddt, id, p.bf16) * sigmoid_f(ld_io(a.z, id, p.bf16) + a.bias[h]);
        st_io(a.dz, id, dz, p.bf16);
        acc += dz;
        if (p.two_ep && a.dlam_logit) {
            const long long il = ix_lam(p, b, t, h);
            const float s = sigmoid_f(ld_io(a.lam_logit, il, p.bf16));
            st_io(a.dlam_logit, il, ld_io(a.dlam, il, p.bf16) * s * (1.f - s), p.bf16);
        }
    }
    red[tid] = acc;
    __syncthreads();
    for (int s = 128; s >= 1; s >>= 1) {
        if (tid < s) red[tid] += red[tid + s];
        __syncthreads();
    }
    if (tid == 0 && a.dbias) a.dbias[h] = red[0];
}

cudaError_t preact_forward(const Params &p, const PreactArgs &a, cudaStream_t st) {
    const long long total = (long long)p.Bsz * p.L * p.H;
    long long blocks = (total + 255) / 256;
    if (blocks > 148 * 16) blocks = 148 * 16;
    if (blocks < 1) blocks = 1;
    k_preact_fwd<<<(int)blocks, 256, 0, st>>>(p, a);
    profile_mark(st, "k_preact_fwd");
    return cudaGetLastError();
}

cudaError_t preact_backward(const Params &p, const PreactArgs &a, cudaStream_t st) {
    k_preact_bwd<<<p.H, 256, 0, st>>>(p, a);
    profile_mark(st, "k_preact_bwd");
    return cudaGetLastError();
}

}  // namespace ssm
