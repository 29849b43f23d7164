// The mixer's output gate around the scan: y_g = y * silu(z), silu(z) = z sigmoid(z),
// z in y's layout.  The pages' fused kernel merges the state update with the gating
// and the output projection of the mixer ("Diagonal Equivalence in State Space
// Models", kongchang.com: the kernel-performance paragraph).  These elementwise passes
// apply it right after the scan's forward, while y is still in L2 (inside the
// instruction-bound tensor-core epilogue it was measured slower), and take its
// gradient (backward):
//     dy = dy_g silu(z),   dz = dy_g y sigmoid(z) (1 + z (1 - sigmoid(z))).
#include "common.cuh"

namespace ssm {

__device__ __forceinline__ float gate_sigmoid(float z) { return __frcp_rn(1.f + __expf(-z)); }

// (b, t, h, o, q) of flat element i of [B][L][H][O][P]
__device__ __forceinline__ long long gate_index(const Params &p, long long i, long long total) {
    int q, o, h, t, b;
    if (total <= 0x7fffffffLL) {
        unsigned r = (unsigned)i;
        q = (int)(r % (unsigned)p.P);
        r /= (unsigned)p.P;
        o = (int)(r % (unsigned)p.O);
        r /= (unsigned)p.O;
        h = (int)(r % (unsigned)p.H);
        r /= (unsigned)p.H;
        t = (int)(r % (unsigned)p.L);
        b = (int)(r / (unsigned)p.L);
    } else {
        long long r = i;
        q = (int)(r % p.P);
        r /= p.P;
        o = (int)(r % p.O);
        r /= p.O;
        h = (int)(r % p.H);
        r /= p.H;
        t = (int)(r % p.L);
        b = (int)(r / p.L);
    }
    return ix_y(p, b, t, h, o, q);
}

// y (the scan's output, in p.y) -> y * silu(z) in place, the pre-gate y copied to
// p.ypre when set.  `vec`: dense layouts and 16-byte aligned tensors, 16 bytes per
// access.
__global__ void __launch_bounds__(256) k_gate_fwd(Params p, int vec) {
    if (gated_off(p)) return;
    const long long total = (long long)p.Bsz * p.L * p.H * p.O * p.P;
    const long long stride = (long long)gridDim.x * blockDim.x;
    if (vec) {
        const int per = p.bf16 ? 8 : 4;   // elements per 16 bytes
        const long long nv = total / per;
        for (long long v = blockIdx.x * (long long)blockDim.x + threadIdx.x; v < nv; v += stride) {
            const uint4 yw = reinterpret_cast<const uint4 *>(p.y)[v];
            const uint4 zw = reinterpret_cast<const uint4 *>(p.gz)[v];
            if (p.ypre) reinterpret_cast<uint4 *>(p.ypre)[v] = yw;
            uint32_t yu[4] = {yw.x, yw.y, yw.z, yw.w}, zu[4] = {zw.x, zw.y, zw.z, zw.w}, o[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                if (p.bf16) {
                    const float y0 = __uint_as_float(yu[k] << 16), y1 = __uint_as_float(yu[k] & 0xffff0000u);
                    const float z0 = __uint_as_float(zu[k] << 16), z1 = __uint_as_float(zu[k] & 0xffff0000u);
                    const __nv_bfloat162 r = __floats2bfloat162_rn(y0 * z0 * gate_sigmoid(z0),
                                                                   y1 * z1 * gate_sigmoid(z1));
                    o[k] = *reinterpret_cast<const uint32_t *>(&r);
                } else {
                    const float y = __uint_as_float(yu[k]), z = __uint_as_float(zu[k]);
                    o[k] = __float_as_uint(y * z * gate_sigmoid(z));
                }
            }
            reinterpret_cast<uint4 *>(p.y)[v] = make_uint4(o[0], o[1], o[2], o[3]);
        }
        return;
    }
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total; i += stride) {
        const long long ix = gate_index(p, i, total);
        const float y = ld_io(p.y, ix, p.bf16), z = ld_io(p.gz, ix, p.bf16);
        if (p.ypre) st_io(p.ypre, ix, y, p.bf16);
        st_io(p.y, ix, y * z * gate_sigmoid(z), p.bf16);
    }
}

__global__ void __launch_bounds__(256) k_gate_bwd(Params p, const void *dyg, void *dy, void *dz) {
    const long long total = (long long)p.Bsz * p.L * p.H * p.O * p.P;
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
         i += (long long)gridDim.x * blockDim.x) {
        const long long ix = gate_index(p, i, total);
        const float g = ld_io(dyg, ix, p.bf16), y = ld_io(p.ypre, ix, p.bf16);
        const float z = ld_io(p.gz, ix, p.bf16), s = gate_sigmoid(z);
        st_io(dz, ix, g * y * s * fmaf(z, 1.f - s, 1.f), p.bf16);
        st_io(dy, ix, g * z * s, p.bf16);
    }
}

static int gate_blocks(const Params &p) {
    const long long total = (long long)p.Bsz * p.L * p.H * p.O * p.P;
    long long b = (total + 255) / 256;
    if (b > 148 * 16) b = 148 * 16;
    return b < 1 ? 1 : (int)b;
}

// dense [B][L][H][O][P] with 16-byte aligned tensors and a whole number of 16-byte pieces
static int gate_vec(const Params &p) {
    const long long P = p.P, OP = (long long)p.O * P, HOP = p.H * OP, LHOP = p.L * HOP;
    const long long total = p.Bsz * LHOP;
    const int per = p.bf16 ? 8 : 4;
    auto a16 = [](const void *q) { return q == nullptr || ((uintptr_t)q & 15) == 0; };
    return p.sy[2] == OP && p.sy[1] == HOP && p.sy[0] == LHOP && total % per == 0 && a16(p.y) &&
           a16(p.gz) && a16(p.ypre);
}

cudaError_t gate_forward(const Params &p, cudaStream_t st) {
    k_gate_fwd<<<gate_blocks(p), 256, 0, st>>>(p, gate_vec(p));
    profile_mark(st, "k_gate_fwd");
    return cudaGetLastError();
}

cudaError_t gate_backward(const Params &p, const void *dyg, void *dy, void *dz, cudaStream_t st) {
    k_gate_bwd<<<gate_blocks(p), 256, 0, st>>>(p, dyg, dy, dz);
    profile_mark(st, "k_gate_bwd");
    return cudaGetLastError();
}

}  // namespace ssm
