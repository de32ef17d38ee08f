// Per-token absmax int8 activation quantisation.
//
// Sparse-BitNet Guide: 1.58-Bit LLMs Meet 2:4 Sparsity, "Mathematical
// Formulation of Sparse-BitLinear", activation equation: beta = max_j |x_j|
// per token, x_q = clip(round(x * 127 / beta), -128, 127); epsilon clamp as in
// the guide's module listing.  Decisions are taken in float32: s = 127 / beta
// is an IEEE division, x * s an IEEE product, round() is half-to-even.
//
// One warp per token.  Pass 1: max of |x| on the bf16 bit patterns (the
// magnitude bits order like the values).  Pass 2: quantise 16-element blocks;
// INTERLEAVED output stores each block as byte 4j + b <- element 4b + j (the
// order in which the contraction kernels expand 2-bit weight codes).
#include "sbl_common.cuh"

namespace sbl {

constexpr int kQuantWarps = 8;

__device__ __forceinline__ int quant1(uint32_t bf16_bits, float s) {
    const float x = __uint_as_float(bf16_bits << 16);
    const int q = __float2int_rn(__fmul_rn(x, s));
    return max(-128, min(127, q));
}

template <bool INTERLEAVED>
__global__ void __launch_bounds__(kQuantWarps * 32) quant_kernel(const uint16_t* __restrict__ x, long long T,
                                                                 long long K, int8_t* __restrict__ xq,
                                                                 float* __restrict__ s_tok, unsigned* status) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long t = static_cast<long long>(blockIdx.x) * kQuantWarps + warp;
    if (t >= T) return;
    const uint4* xr = reinterpret_cast<const uint4*>(x + t * K);
    const int nvec = static_cast<int>(K >> 3);  // 8 bf16 per 16-byte vector

    uint32_t mx = 0;
    for (int v = lane; v < nvec; v += 32) {
        const uint4 u = ldg_nc(xr + v);
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            mx = max(mx, w[i] & 0x7FFFu);
            mx = max(mx, (w[i] >> 16) & 0x7FFFu);
        }
    }
    mx = __reduce_max_sync(0xFFFFFFFFu, mx);
    if (mx >= 0x7F80u && lane == 0) raise_status(status, kStatusNonfinite);
    const float amax = __uint_as_float(mx << 16);
    const float s = __fdiv_rn(127.0f, fmaxf(amax, 1e-5f));
    if (lane == 0) s_tok[t] = s;

    int8_t* out = xq + t * K;
    const int nblk = static_cast<int>(K >> 4);
    for (int b = lane; b < nblk; b += 32) {
        const uint4 u0 = ldg_nc(xr + 2 * b);
        const uint4 u1 = ldg_nc(xr + 2 * b + 1);
        const uint32_t w[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
        int q[16];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            q[2 * i] = quant1(w[i] & 0xFFFFu, s);
            q[2 * i + 1] = quant1(w[i] >> 16, s);
        }
        uint32_t o[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            uint32_t word = 0;
#pragma unroll
            for (int bb = 0; bb < 4; ++bb) {
                const int src = INTERLEAVED ? (4 * bb + j) : (4 * j + bb);
                word |= (static_cast<uint32_t>(q[src]) & 0xFFu) << (8 * bb);
            }
            o[j] = word;
        }
        *reinterpret_cast<uint4*>(out + 16 * b) = make_uint4(o[0], o[1], o[2], o[3]);
    }
}

cudaError_t launch_quant(const uint16_t* x, long long T, long long K, int8_t* xq, float* s_tok, bool interleaved,
                         unsigned* status, cudaStream_t stream) {
    const unsigned blocks = static_cast<unsigned>((T + kQuantWarps - 1) / kQuantWarps);
    if (interleaved)
        quant_kernel<true><<<blocks, kQuantWarps * 32, 0, stream>>>(x, T, K, xq, s_tok, status);
    else
        quant_kernel<false><<<blocks, kQuantWarps * 32, 0, stream>>>(x, T, K, xq, s_tok, status);
    return cudaGetLastError();
}

}  // namespace sbl
