// Straight-through (STE) backward of the Sparse-BitLinear layer: the training
// path's two gradient contractions over the packed weights.
//
// The guide's "Training Stability & The Straight-Through Estimator" lets the
// gradient pass the N:M mask and the ternary rounding unchanged to the latent
// weights, and the Sparse-BitNet README ("How It Works / BitLinear") passes it
// through the quantiser the same way; with the activation quantiser passed
// through as well, the forward reads y = x_hat . W_hat^T with
// x_hat[t,k] = x_q[t,k] / s_t and W_hat[o,k] = scale_o * W_t[o,k], so
//     dX [T, K] = dY . W_hat        (contraction over O)
//     dW [O, K] = dY^T . x_hat      (contraction over T, every position)
// and, for the guide module's form (the gradient taken at the ternary matrix
// of y = (x~ . W~^T) * beta * gamma / 127), dW row o scaled by scale_o.
//
// Both are float contractions of a float operand (dY, with the row or token
// scale folded in as it is staged) against a small-integer operand (2-bit
// ternary codes decoded while staging, or int8 activations), accumulated in
// fp32 with fused multiply-adds: the products with {-1, 0, 1} or an int8 are
// exact up to the fma's single rounding, so every output is within
// (n + 2) * 2^-24 * sum |terms| of the exact value for a reduction of length n
// ((n + 3) with the extra row-scale product of the ternary form).
// One CTA computes a 128 x 128 output tile C[i, j] = sum_r A[r, i] * B[r, j]
// on the CUDA cores (16 x 16 threads, 8 x 8 outputs each), staging 16-deep
// slices of A and B in two shared-memory buffers: the next slice is loaded
// into registers while the current one is multiplied.  Bounded by fp32 FMA
// issue, not by HBM: per tile 2 * 128 * 128 * n flops against
// (128 + 128) * n operand elements.
#include "sbl_common.cuh"

namespace sbl {

constexpr int kBwTile = 128;         // output tile edge (rows i, columns j = k)
constexpr int kBwR = 16;             // reduction slice per stage
constexpr int kBwThreads = 256;      // 16 x 16 threads
constexpr int kBwLd = kBwTile + 4;   // shared row pitch in floats (16-byte rows, spread banks)
constexpr int kBwdDx = 0, kBwdDw = 1;

// Ternary value of 2-bit code c (00 = 0, 01 = +1, 10 = -1; 11 never written, read as 0).
__device__ __forceinline__ float code_value(uint32_t c) {
    return static_cast<float>(static_cast<int>(c & 1u) - static_cast<int>(c >> 1));
}

// MODE kBwdDx: rows i = tokens t, reduction r = output rows o,
//   A[r, i] = dY[t, o] * scale_o, B[r, j] = W_t[o, k].
// MODE kBwdDw: rows i = output rows o, reduction r = tokens t,
//   A[r, i] = dY[t, o] / s_t, B[r, j] = x_q[t, k].
// out is row-major [rows, K].  Tiles are numbered row-tile-major over
// tiles_j column tiles.
template <int MODE>
__global__ void __launch_bounds__(kBwThreads, 2)
ste_backward_kernel(const float* __restrict__ dY, long long T, long long O, long long K,
                    const uint8_t* __restrict__ packed, const float* __restrict__ row_scale,
                    const int8_t* __restrict__ xq, const float* __restrict__ s_tok, float* __restrict__ out,
                    int dw_ternary, long long tiles_j) {
    __shared__ __align__(16) float sa[2][kBwR][kBwLd];
    __shared__ __align__(16) float sb[2][kBwR][kBwLd];
    const int tid = threadIdx.x;
    const long long i0 = static_cast<long long>(blockIdx.x / tiles_j) * kBwTile;
    const long long j0 = static_cast<long long>(blockIdx.x % tiles_j) * kBwTile;
    const long long rows = MODE == kBwdDx ? T : O;
    const long long red = MODE == kBwdDx ? O : T;
    const long long nst = (red + kBwR - 1) / kBwR;

    // Operand staging registers: 8 elements of A, one 16-element piece of B
    // (threads 0..127: slice row tid / 8, columns 16 * (tid % 8) .. + 15).
    float ra[8];
    uint4 rb = make_uint4(0u, 0u, 0u, 0u);
    const int br = tid >> 3, bj = (tid & 7) * 16;

    // dX: this thread's A elements come from tokens i0 + tid/16 + 16 q, q < qn.
    const long long t_first = i0 + (tid >> 4);
    const int qn = MODE == kBwdDx ? static_cast<int>(t_first < T ? min(8ll, (T - t_first + 15) / 16) : 0ll) : 0;
    const float* dy_row = dY + (MODE == kBwdDx ? t_first * O : i0 + (tid & 127));

    auto load = [&](long long r0) {
        if constexpr (MODE == kBwdDx) {
            // element q: r = tid % 16, i = tid / 16 + 16 q (16 consecutive o of one token per half-warp)
            const long long o = r0 + (tid & 15);
            const bool ok = o < O;
            const float sc = ok ? __ldg(row_scale + o) : 0.0f;
            const float* p = dy_row + o;
#pragma unroll
            for (int q = 0; q < 8; ++q) ra[q] = (ok && q < qn) ? __fmul_rn(__ldg(p + q * 16 * O), sc) : 0.0f;
            if (tid < 128) {
                const long long orow = r0 + br;
                rb.x = (orow < O && j0 + bj < K)
                           ? __ldg(reinterpret_cast<const uint32_t*>(packed + orow * (K / 4) + (j0 + bj) / 4))
                           : 0u;
            }
        } else {
            // element q: i = tid % 128, r = tid / 128 + 2 q (a warp reads 32 consecutive o of one token)
            const bool ok = i0 + (tid & 127) < O;
            const long long t1 = r0 + (tid >> 7);
            const float* p = dy_row + t1 * O;
#pragma unroll
            for (int q = 0; q < 8; ++q)
                ra[q] = (ok && t1 + 2 * q < T) ? __fdiv_rn(__ldg(p + q * 2 * O), __ldg(s_tok + t1 + 2 * q)) : 0.0f;
            if (tid < 128) {
                const long long t = r0 + br;
                rb = (t < T && j0 + bj < K) ? __ldg(reinterpret_cast<const uint4*>(xq + t * K + j0 + bj))
                                            : make_uint4(0u, 0u, 0u, 0u);
            }
        }
    };
    auto store = [&](int st) {
        if constexpr (MODE == kBwdDx) {
#pragma unroll
            for (int q = 0; q < 8; ++q) sa[st][tid & 15][(tid >> 4) + 16 * q] = ra[q];
        } else {
#pragma unroll
            for (int q = 0; q < 8; ++q) sa[st][(tid >> 7) + 2 * q][tid & 127] = ra[q];
        }
        if (tid < 128) {
            float v[16];
            if constexpr (MODE == kBwdDx) {
#pragma unroll
                for (int q = 0; q < 16; ++q) v[q] = code_value((rb.x >> (2 * q)) & 3u);
            } else {
                const uint32_t w[4] = {rb.x, rb.y, rb.z, rb.w};
#pragma unroll
                for (int q = 0; q < 16; ++q)
                    v[q] = static_cast<float>(static_cast<int8_t>((w[q >> 2] >> (8 * (q & 3))) & 0xFFu));
            }
            float4* dst = reinterpret_cast<float4*>(&sb[st][br][bj]);
#pragma unroll
            for (int q = 0; q < 4; ++q) dst[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
        }
    };

    const int tx = tid & 15, ty = tid >> 4;
    float acc[8][8];
#pragma unroll
    for (int a = 0; a < 8; ++a)
#pragma unroll
        for (int b = 0; b < 8; ++b) acc[a][b] = 0.0f;

    if (nst > 0) {
        load(0);
        store(0);
        __syncthreads();
    }
    for (long long c = 0; c < nst; ++c) {
        const int st = static_cast<int>(c & 1);
        if (c + 1 < nst) load((c + 1) * kBwR);
#pragma unroll
        for (int r = 0; r < kBwR; ++r) {
            const float4 a0 = *reinterpret_cast<const float4*>(&sa[st][r][ty * 4]);
            const float4 a1 = *reinterpret_cast<const float4*>(&sa[st][r][64 + ty * 4]);
            const float4 b0 = *reinterpret_cast<const float4*>(&sb[st][r][tx * 4]);
            const float4 b1 = *reinterpret_cast<const float4*>(&sb[st][r][64 + tx * 4]);
            const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
            const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
            for (int a = 0; a < 8; ++a)
#pragma unroll
                for (int b = 0; b < 8; ++b) acc[a][b] = __fmaf_rn(av[a], bv[b], acc[a][b]);
        }
        if (c + 1 < nst) store(st ^ 1);
        __syncthreads();
    }

    // Epilogue: rows ty*4 + a (a < 4) and 64 + ty*4 + a - 4; columns tx*4.. and 64 + tx*4..
    // K % 16 == 0, so a 4-column group lies wholly inside or outside the matrix.
#pragma unroll
    for (int a = 0; a < 8; ++a) {
        const long long row = i0 + (a < 4 ? ty * 4 + a : 64 + ty * 4 + a - 4);
        if (row >= rows) continue;
        const float sc = (MODE == kBwdDw && dw_ternary) ? __ldg(row_scale + row) : 1.0f;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const long long col = j0 + h * 64 + tx * 4;
            if (col >= K) continue;
            float4 v = make_float4(acc[a][4 * h], acc[a][4 * h + 1], acc[a][4 * h + 2], acc[a][4 * h + 3]);
            if (MODE == kBwdDw && dw_ternary) {
                v.x = __fmul_rn(v.x, sc);
                v.y = __fmul_rn(v.y, sc);
                v.z = __fmul_rn(v.z, sc);
                v.w = __fmul_rn(v.w, sc);
            }
            *reinterpret_cast<float4*>(out + row * K + col) = v;
        }
    }
}

// Output tiles of one gradient (0 when it is empty).
long long ste_backward_tiles(long long rows, long long K) {
    return ((rows + kBwTile - 1) / kBwTile) * ((K + kBwTile - 1) / kBwTile);
}

// dX (may be null): dY . (scale * W_t); dW (may be null): dY^T . (x_q / s_t),
// scaled by row_scale per row when dw_ternary.  Sizes and pointers are checked
// by the caller; K % 16 == 0, every tile count below 2^31.
cudaError_t launch_ste_backward(const float* dY, long long T, long long O, long long K, const uint8_t* packed,
                                const float* row_scale, const int8_t* xq, const float* s_tok, float* dX, float* dW,
                                int dw_ternary, cudaStream_t stream) {
    const long long tj = (K + kBwTile - 1) / kBwTile;
    if (dX) {
        const long long tiles = ste_backward_tiles(T, K);
        if (tiles > 0)
            ste_backward_kernel<kBwdDx><<<static_cast<unsigned>(tiles), kBwThreads, 0, stream>>>(
                dY, T, O, K, packed, row_scale, xq, s_tok, dX, 0, tj);
    }
    if (dW) {
        const long long tiles = ste_backward_tiles(O, K);
        if (tiles > 0)
            ste_backward_kernel<kBwdDw><<<static_cast<unsigned>(tiles), kBwThreads, 0, stream>>>(
                dY, T, O, K, packed, row_scale, xq, s_tok, dW, dw_ternary, tj);
    }
    return cudaGetLastError();
}

}  // namespace sbl
