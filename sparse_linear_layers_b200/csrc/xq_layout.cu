// Quantised activations from column order into the pairing order.
//
// sbl_linear_q contracts activations that the caller quantised already
// (sbl_quant_act: int8 x_q in column order and s_tok per token; Sparse-BitNet
// Guide, "Mathematical Formulation of Sparse-BitLinear", the activation
// equation).  The tensor-core GEMMs and the warp-MMA decode read x_q in the
// order in which expand_pairs() unpacks the weight codes: within each block of
// 16 activations the even elements 0..6, the odd 1..7, the even 8..14, the odd
// 9..15.  This kernel is that byte permutation and nothing else: four byte
// permutes per 16-byte block, HBM-bound (T * K bytes read and written).
//
// It is a programmatic dependent of its predecessor (which may still be
// writing x_q) and signals its own dependents at entry, like the quantisation
// kernel it stands in for.
#include "sbl_common.cuh"

namespace sbl {

__global__ void __launch_bounds__(256) xq_to_pairs_kernel(const uint4* __restrict__ in, uint4* __restrict__ out,
                                                          long long n16) {
    asm volatile("griddepcontrol.launch_dependents;");
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
    for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < n16; i += stride) {
        const uint4 v = ldg_nc(in + i);  // bytes 0..3 in v.x, 4..7 in v.y, ...
        out[i] = make_uint4(prmt(v.x, v.y, 0x6420u), prmt(v.x, v.y, 0x7531u), prmt(v.z, v.w, 0x6420u),
                            prmt(v.z, v.w, 0x7531u));
    }
}

// T x K int8 (K % 16 == 0, both pointers 16-byte aligned): at most eight
// blocks of 256 threads per SM, grid-stride beyond that.
cudaError_t launch_xq_to_pairs(const int8_t* xq, long long T, long long K, int8_t* out, int num_sms,
                               cudaStream_t stream) {
    const long long n16 = T * (K / 16);
    if (n16 <= 0) return cudaSuccess;
    long long blocks = (n16 + 255) / 256;
    const long long cap = 8LL * (num_sms > 0 ? num_sms : 1);
    if (blocks > cap) blocks = cap;
    return pdl_launch(xq_to_pairs_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, stream,
                      reinterpret_cast<const uint4*>(xq), reinterpret_cast<uint4*>(out), n16);
}

}  // namespace sbl
