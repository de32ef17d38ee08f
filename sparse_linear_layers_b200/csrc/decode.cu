// Decode path: y = dequant(x_q . W_t^T) for a handful of tokens on CUDA cores.
//
// The integer product of the Sparse-BitNet Guide's linear-evaluation equation
// ("Mathematical Formulation of Sparse-BitLinear") for small T is a stream over
// the 2-bit weights (0.25 B per weight, read once), so it is bound by HBM
// bandwidth; the guide notes that memory bandwidth decides serving cost.
//
// Layout: a row of packed weights is K/4 bytes = CPR chunks of CW 32-bit words
// (16 CW weights; CW = 4 when K % 64 == 0 so rows are 16-byte aligned, else
// CW = 1).  L lanes share a row (32/L rows per warp); lane li of a row takes
// chunks li, li+L, ...  Each chunk is one streaming load.
// Activations (already quantised, interleaved in 16-element blocks) sit in
// shared memory as xs[t][word][chunk] 16-byte units, so the L lanes of a row
// read consecutive units (no bank conflicts) and rows of one warp read the
// same units (broadcast).
//
// Arithmetic per 32-bit weight word (16 weights): for j = 0..3 the masks
// w & (0x01010101 << 2j) and w & (0x02020202 << 2j) pick the +1 and -1 codes
// of weights 4b + j (scaled by 4^j and 2*4^j); one unsigned-by-signed dp4a each
// against the interleaved activation word j accumulates them.  The scales are
// removed exactly (every partial is a multiple of its power of two) before the
// L-lane shuffle reduction.
#include "sbl_common.cuh"

namespace sbl {

constexpr int kDecodeThreads = 256;

template <int L, int TT, int CW>
__global__ void __launch_bounds__(kDecodeThreads) decode_kernel(const uint8_t* __restrict__ packed,
                                                                const float* __restrict__ row_scale, long long O,
                                                                int K, const int8_t* __restrict__ xperm,
                                                                const float* __restrict__ s_tok, long long T,
                                                                long long t0, void* __restrict__ y, int y_bf16,
                                                                int32_t* __restrict__ acc_out) {
    extern __shared__ uint4 xs[];
    const int CPR = K / (16 * CW);
    const int units = TT * CW * CPR;
    for (int i = threadIdx.x; i < units; i += blockDim.x) {
        const int t = i / (CW * CPR);
        const int r = i - t * CW * CPR;
        const int c = r / CW, w = r % CW;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (t0 + t < T) v = ldg_nc(xperm + (t0 + t) * K + 16 * (CW * c + w));
        xs[(t * CW + w) * CPR + c] = v;
    }
    __syncthreads();

    constexpr int RW = 32 / L;
    const int lane = threadIdx.x & 31;
    const int sub = lane / L, li = lane % L;
    const long long gw = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const long long nw = (static_cast<long long>(gridDim.x) * blockDim.x) >> 5;
    const long long ngroups = (O + RW - 1) / RW;

    for (long long g = gw; g < ngroups; g += nw) {
        const long long row = g * RW + sub;
        const bool valid = row < O;
        int alo[TT][4], ahi[TT][4];
#pragma unroll
        for (int t = 0; t < TT; ++t)
#pragma unroll
            for (int j = 0; j < 4; ++j) alo[t][j] = ahi[t][j] = 0;
        if (valid) {
            const uint8_t* prow = packed + row * (K >> 2);
#pragma unroll 2
            for (int c = li; c < CPR; c += L) {
                uint32_t ww[CW];
                if constexpr (CW == 4) {
                    const uint4 wv = ldg_stream(prow + 16 * c);
                    ww[0] = wv.x; ww[1 % CW] = wv.y; ww[2 % CW] = wv.z; ww[3 % CW] = wv.w;
                } else {
                    ww[0] = __ldg(reinterpret_cast<const unsigned int*>(prow) + c);
                }
#pragma unroll
                for (int w = 0; w < CW; ++w) {
                    uint32_t mlo[4], mhi[4];
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        mlo[j] = ww[w] & (0x01010101u << (2 * j));
                        mhi[j] = ww[w] & (0x02020202u << (2 * j));
                    }
#pragma unroll
                    for (int t = 0; t < TT; ++t) {
                        const uint4 xv = xs[(t * CW + w) * CPR + c];
                        const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            alo[t][j] = dp4a_us(mlo[j], xw[j], alo[t][j]);
                            ahi[t][j] = dp4a_us(mhi[j], xw[j], ahi[t][j]);
                        }
                    }
                }
            }
        }
        int acc[TT];
#pragma unroll
        for (int t = 0; t < TT; ++t) {
            int a = 0;
#pragma unroll
            for (int j = 0; j < 4; ++j) a += (alo[t][j] >> (2 * j)) - (ahi[t][j] >> (2 * j + 1));
#pragma unroll
            for (int off = L / 2; off >= 1; off >>= 1) a += __shfl_xor_sync(0xFFFFFFFFu, a, off);
            acc[t] = a;
        }
        if (valid && li == 0) {
            const float sc = row_scale[row];
#pragma unroll
            for (int t = 0; t < TT; ++t) {
                const long long tt = t0 + t;
                if (tt < T) {
                    const float v = __fdiv_rn(__fmul_rn(static_cast<float>(acc[t]), sc), s_tok[tt]);
                    if (y_bf16)
                        reinterpret_cast<__nv_bfloat16_raw*>(y)[tt * O + row] =
                            static_cast<__nv_bfloat16_raw>(__float2bfloat16_rn(v));
                    else
                        reinterpret_cast<float*>(y)[tt * O + row] = v;
                    if (acc_out) acc_out[tt * O + row] = acc[t];
                }
            }
        }
    }
}

// Lanes per row: best chunk utilisation, weighted by how well the warp count
// fills the GPU (small layers prefer wide rows, large ones exact fits).
static int choose_lanes(long long O, int cpr, int num_sms) {
    int best = 32;
    double best_score = -1.0;
    for (int L = 32; L >= 1; L >>= 1) {
        const double eff = static_cast<double>(cpr) / (static_cast<double>((cpr + L - 1) / L) * L);
        const double warps = static_cast<double>((O + (32 / L) - 1) / (32 / L));
        const double fill = warps / (num_sms * 16.0);
        const double score = eff * (fill < 1.0 ? fill : 1.0);
        if (score > best_score + 1e-9) {
            best_score = score;
            best = L;
        }
    }
    return best;
}

template <int L, int TT, int CW>
static cudaError_t launch_decode_lt(const uint8_t* packed, const float* row_scale, long long O, int K,
                                    const int8_t* xperm, const float* s_tok, long long T, long long t0, void* y,
                                    int y_bf16, int32_t* acc_out, int num_sms, cudaStream_t stream) {
    const size_t smem = static_cast<size_t>(TT) * K;
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(decode_kernel<L, TT, CW>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(smem));
        if (e != cudaSuccess) return e;
    }
    constexpr int RW = 32 / L;
    const long long groups = (O + RW - 1) / RW;
    const long long warps_per_block = kDecodeThreads / 32;
    long long blocks = (groups + warps_per_block - 1) / warps_per_block;
    const long long cap = static_cast<long long>(num_sms) * 4;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    decode_kernel<L, TT, CW><<<static_cast<unsigned>(blocks), kDecodeThreads, smem, stream>>>(
        packed, row_scale, O, K, xperm, s_tok, T, t0, y, y_bf16, acc_out);
    return cudaGetLastError();
}

template <int TT, int CW>
static cudaError_t launch_decode_t(int L, const uint8_t* packed, const float* row_scale, long long O, int K,
                                   const int8_t* xperm, const float* s_tok, long long T, long long t0, void* y,
                                   int y_bf16, int32_t* acc_out, int num_sms, cudaStream_t stream) {
    switch (L) {
        case 32: return launch_decode_lt<32, TT, CW>(packed, row_scale, O, K, xperm, s_tok, T, t0, y, y_bf16, acc_out, num_sms, stream);
        case 16: return launch_decode_lt<16, TT, CW>(packed, row_scale, O, K, xperm, s_tok, T, t0, y, y_bf16, acc_out, num_sms, stream);
        case 8: return launch_decode_lt<8, TT, CW>(packed, row_scale, O, K, xperm, s_tok, T, t0, y, y_bf16, acc_out, num_sms, stream);
        case 4: return launch_decode_lt<4, TT, CW>(packed, row_scale, O, K, xperm, s_tok, T, t0, y, y_bf16, acc_out, num_sms, stream);
        case 2: return launch_decode_lt<2, TT, CW>(packed, row_scale, O, K, xperm, s_tok, T, t0, y, y_bf16, acc_out, num_sms, stream);
        default: return launch_decode_lt<1, TT, CW>(packed, row_scale, O, K, xperm, s_tok, T, t0, y, y_bf16, acc_out, num_sms, stream);
    }
}

template <int TT>
static cudaError_t launch_decode_cw(int L, bool wide, const uint8_t* packed, const float* row_scale, long long O,
                                    int K, const int8_t* xperm, const float* s_tok, long long T, long long t0,
                                    void* y, int y_bf16, int32_t* acc_out, int num_sms, cudaStream_t stream) {
    if (wide)
        return launch_decode_t<TT, 4>(L, packed, row_scale, O, K, xperm, s_tok, T, t0, y, y_bf16, acc_out, num_sms, stream);
    return launch_decode_t<TT, 1>(L, packed, row_scale, O, K, xperm, s_tok, T, t0, y, y_bf16, acc_out, num_sms, stream);
}

// Decode for any T: passes of up to 8 tokens (later passes re-read the
// weights, mostly from L2).  Needs K % 16 == 0.
cudaError_t launch_decode(const uint8_t* packed, const float* row_scale, long long O, long long K,
                          const int8_t* xperm, const float* s_tok, long long T, void* y, int y_bf16,
                          int32_t* acc_out, int num_sms, cudaStream_t stream) {
    const int Ki = static_cast<int>(K);
    const bool wide = (Ki % 64) == 0;
    const int cpr = wide ? Ki / 64 : Ki / 16;
    const int L = choose_lanes(O, cpr, num_sms);
    for (long long t0 = 0; t0 < T; t0 += 8) {
        const long long rem = T - t0;
        cudaError_t e;
        if (rem > 4) e = launch_decode_cw<8>(L, wide, packed, row_scale, O, Ki, xperm, s_tok, T, t0, y, y_bf16, acc_out, num_sms, stream);
        else if (rem > 2) e = launch_decode_cw<4>(L, wide, packed, row_scale, O, Ki, xperm, s_tok, T, t0, y, y_bf16, acc_out, num_sms, stream);
        else if (rem == 2) e = launch_decode_cw<2>(L, wide, packed, row_scale, O, Ki, xperm, s_tok, T, t0, y, y_bf16, acc_out, num_sms, stream);
        else e = launch_decode_cw<1>(L, wide, packed, row_scale, O, Ki, xperm, s_tok, T, t0, y, y_bf16, acc_out, num_sms, stream);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace sbl
