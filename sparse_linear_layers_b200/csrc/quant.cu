// Per-token absmax int8 activation quantisation.
//
// Sparse-BitNet Guide: 1.58-Bit LLMs Meet 2:4 Sparsity, "Mathematical
// Formulation of Sparse-BitLinear", activation equation: beta = max_j |x_j|
// per token, x_q = clip(round(x * 127 / beta), -128, 127); epsilon clamp as in
// the guide's module listing.  Decisions are taken in float32: s = 127 / beta
// is an IEEE division, x * s an IEEE product, round() is half-to-even.
//
// TPT threads share a token; each holds up to BPT 16-element blocks in
// registers, so x is read once.  The max of |x| is taken on the bf16 bit
// patterns (magnitude bits order like the values).  Output layouts:
//   NATURAL      x_q in column order (the public sbl_quant_act);
//   PAIRS        each 16-element block stored as its even elements 0..6, odd
//                elements 1..7, even 8..14, odd 9..15: the order in which the
//                tensor-core kernels expand weight codes (expand_pairs; read
//                by TMA).
// The kernel signals programmatic dependents at entry: the contraction kernel
// that follows may start its own prologue while this one runs.
#include "sbl_common.cuh"

namespace sbl {

enum QuantLayout { kNatural = 0, kPairs = 1 };

template <int LAYOUT>
__device__ __forceinline__ void quant_block_store(const uint4& u0, const uint4& u1, float s, int8_t* out_row, int b,
                                                  long long K) {
    (void)K;
    *reinterpret_cast<uint4*>(out_row + 16 * static_cast<long long>(b)) =
        LAYOUT == kNatural ? quant_block16<false>(u0, u1, s) : quant_block16_pairs(u0, u1, s);
}

// Zero `n16` 16-byte words at p, spread over the whole grid.
__device__ __forceinline__ void zero_fill(uint4* p, long long n16) {
    const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
    for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < n16; i += stride)
        p[i] = make_uint4(0u, 0u, 0u, 0u);
}

// Register-resident variant: K / 16 <= TPT * BPT.
template <int LAYOUT, int TPT, int BPT>
__global__ void __launch_bounds__(256) quant_kernel(const uint16_t* __restrict__ x, long long T, long long K,
                                                    int8_t* __restrict__ xq, float* __restrict__ s_tok,
                                                    uint4* __restrict__ zero_words, long long nzero, unsigned* status) {
    asm volatile("griddepcontrol.launch_dependents;");
    zero_fill(zero_words, nzero);
    constexpr int TPC = 256 / TPT;
    __shared__ uint32_t red[8];
    const int sub = threadIdx.x / TPT, tr = threadIdx.x % TPT;
    const long long t = static_cast<long long>(blockIdx.x) * TPC + sub;
    const bool valid = t < T;
    const int nblk = static_cast<int>(K >> 4);
    const uint4* xr = reinterpret_cast<const uint4*>(x + (valid ? t : 0) * K);

    uint4 v[BPT][2];
    uint32_t mx = 0;
#pragma unroll
    for (int j = 0; j < BPT; ++j) {
        const int b = tr + TPT * j;
        if (valid && b < nblk) {
            v[j][0] = ldg_nc(xr + 2 * b);
            v[j][1] = ldg_nc(xr + 2 * b + 1);
        } else {
            v[j][0] = v[j][1] = make_uint4(0u, 0u, 0u, 0u);
        }
    }
#pragma unroll
    for (int j = 0; j < BPT; ++j) mx = absmax8(v[j][1], absmax8(v[j][0], mx));
    if constexpr (TPT >= 32) {
        mx = __reduce_max_sync(0xFFFFFFFFu, mx);
    } else {
        // TPT lanes of the warp per token: reduce within each group
#pragma unroll
        for (int off = TPT / 2; off >= 1; off >>= 1) mx = max(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, off));
    }
    if constexpr (TPT > 32) {
        if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = mx;
        __syncthreads();
        const int w0 = sub * (TPT / 32);
#pragma unroll
        for (int i = 0; i < TPT / 32; ++i) mx = max(mx, red[w0 + i]);
    }
    if (!valid) return;
    if (mx >= 0x7F80u && tr == 0) raise_status(status, kStatusNonfinite);
    const float amax = __uint_as_float(mx << 16);
    const float s = __fdiv_rn(127.0f, fmaxf(amax, 1e-5f));
    if (tr == 0) s_tok[t] = s;
    int8_t* out = xq + t * K;
#pragma unroll
    for (int j = 0; j < BPT; ++j) {
        const int b = tr + TPT * j;
        if (b < nblk) quant_block_store<LAYOUT>(v[j][0], v[j][1], s, out, b, K);
    }
}

// Any K: one warp per token, two passes over x (the second mostly from L1/L2).
template <int LAYOUT>
__global__ void __launch_bounds__(256) quant_kernel_loop(const uint16_t* __restrict__ x, long long T, long long K,
                                                         int8_t* __restrict__ xq, float* __restrict__ s_tok,
                                                         uint4* __restrict__ zero_words, long long nzero, unsigned* status) {
    asm volatile("griddepcontrol.launch_dependents;");
    zero_fill(zero_words, nzero);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long t = static_cast<long long>(blockIdx.x) * 8 + warp;
    if (t >= T) return;
    const uint4* xr = reinterpret_cast<const uint4*>(x + t * K);
    const int nvec = static_cast<int>(K >> 3);
    uint32_t mx = 0;
#pragma unroll 4
    for (int v = lane; v < nvec; v += 32) mx = absmax8(ldg_nc(xr + v), mx);
    mx = __reduce_max_sync(0xFFFFFFFFu, mx);
    if (mx >= 0x7F80u && lane == 0) raise_status(status, kStatusNonfinite);
    const float s = __fdiv_rn(127.0f, fmaxf(__uint_as_float(mx << 16), 1e-5f));
    if (lane == 0) s_tok[t] = s;
    const int nblk = static_cast<int>(K >> 4);
#pragma unroll 2
    for (int b = lane; b < nblk; b += 32)
        quant_block_store<LAYOUT>(ldg_nc(xr + 2 * b), ldg_nc(xr + 2 * b + 1), s, xq + t * K, b, K);
}

template <int LAYOUT, int TPT, int BPT>
static void launch_rr(const uint16_t* x, long long T, long long K, int8_t* xq, float* s_tok, uint4* zero_words,
                      long long nzero, unsigned* status, cudaStream_t stream) {
    constexpr int TPC = 256 / TPT;
    const unsigned blocks = static_cast<unsigned>((T + TPC - 1) / TPC);
    quant_kernel<LAYOUT, TPT, BPT><<<blocks, 256, 0, stream>>>(x, T, K, xq, s_tok, zero_words, nzero, status);
}

static int device_sms() {
    static int cached[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    if (!cached[dev] && cudaDeviceGetAttribute(&cached[dev], cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        cached[dev] = 148;
    return cached[dev];
}

template <int LAYOUT>
static cudaError_t launch_layout(const uint16_t* x, long long T, long long K, int8_t* xq, float* s_tok,
                                 uint4* zero_words, long long nzero, unsigned* status, cudaStream_t stream) {
    const long long nblk = K >> 4;
    // Threads per token: the fewest whose registers hold the row (so each thread
    // has up to four 16-element blocks, eight 16-byte loads, in flight), more
    // while the grid would be under two blocks per SM.
    int tpt = 16;
    while (tpt < 256 && tpt * 4 < nblk) tpt *= 2;
    const long long min_blocks = 2LL * device_sms();
    while (tpt < 256 && (T * tpt + 255) / 256 < min_blocks) tpt *= 2;
    if (nblk > 256 * 4) {
        const unsigned blocks = static_cast<unsigned>((T + 7) / 8);
        quant_kernel_loop<LAYOUT><<<blocks, 256, 0, stream>>>(x, T, K, xq, s_tok, zero_words, nzero, status);
    } else if (tpt == 16) {
        launch_rr<LAYOUT, 16, 4>(x, T, K, xq, s_tok, zero_words, nzero, status, stream);
    } else if (tpt == 32) {
        launch_rr<LAYOUT, 32, 4>(x, T, K, xq, s_tok, zero_words, nzero, status, stream);
    } else if (tpt == 64) {
        launch_rr<LAYOUT, 64, 4>(x, T, K, xq, s_tok, zero_words, nzero, status, stream);
    } else if (tpt == 128) {
        launch_rr<LAYOUT, 128, 4>(x, T, K, xq, s_tok, zero_words, nzero, status, stream);
    } else {
        launch_rr<LAYOUT, 256, 4>(x, T, K, xq, s_tok, zero_words, nzero, status, stream);
    }
    return cudaGetLastError();
}

// zero16[0 .. nzero16) (16-byte words) are set to zero as well: the split-K
// accumulators of the contraction that follows.
cudaError_t launch_quant(const uint16_t* x, long long T, long long K, int8_t* xq, float* s_tok, int layout,
                         unsigned* status, cudaStream_t stream, void* zero16, long long nzero16) {
    uint4* zero_words = static_cast<uint4*>(zero16);
    const long long nzero = nzero16;
    switch (layout) {
        case kPairs: return launch_layout<kPairs>(x, T, K, xq, s_tok, zero_words, nzero, status, stream);
        default: return launch_layout<kNatural>(x, T, K, xq, s_tok, zero_words, nzero, status, stream);
    }
}

// ---------------------------------------------------------------- RMSNorm front end
// The guide's SparseBitLinear module normalises x with RMSNorm before the
// per-token absmax ("Mathematical Formulation of Sparse-BitLinear", activation
// step, and the module listing): x_norm = x * (1 / sqrt(mean(x^2) + eps)) * g,
// every step an IEEE float32 operation, then the absmax quantisation above.
// One warp per token; lane l owns the 16-element blocks b with b % 32 == l.
// The sum of squares follows a fixed order: each lane adds its squares in
// increasing k, then an xor butterfly at offsets 16, 8, 4, 2, 1 combines the
// lanes (every lane ends with the same total).  A lane keeps up to RB blocks
// in registers across the three passes (sum of squares, absmax of the
// normalised values, quantisation); blocks beyond that are read again.
template <int LAYOUT>
__global__ void __launch_bounds__(256) rmsnorm_quant_kernel(const uint16_t* __restrict__ x,
                                                            const float* __restrict__ g, float eps, long long T,
                                                            long long K, int8_t* __restrict__ xq,
                                                            float* __restrict__ s_tok, uint4* __restrict__ zero_words,
                                                            long long nzero, unsigned* status) {
    asm volatile("griddepcontrol.launch_dependents;");
    zero_fill(zero_words, nzero);
    constexpr int RB = 4;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long t = static_cast<long long>(blockIdx.x) * 8 + warp;
    if (t >= T) return;
    const uint4* xr = reinterpret_cast<const uint4*>(x + t * K);
    const int nblk = static_cast<int>(K >> 4);
    uint4 v[RB][2];
    // pass 1: sum of squares in the lane's k order; non-finite inputs flagged
    float ss = 0.f;
    uint32_t bad = 0;
    auto add_sq = [&](const uint4& a, const uint4& b) {
        const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float lo = __uint_as_float(w[i] << 16), hi = __uint_as_float(w[i] & 0xFFFF0000u);
            ss = __fadd_rn(ss, __fmul_rn(lo, lo));
            ss = __fadd_rn(ss, __fmul_rn(hi, hi));
            bad |= ((w[i] & 0x7F80u) == 0x7F80u) | ((w[i] & 0x7F800000u) == 0x7F800000u);
        }
    };
#pragma unroll
    for (int j = 0; j < RB; ++j) {
        const int b = lane + 32 * j;
        if (b < nblk) {
            v[j][0] = ldg_nc(xr + 2 * b);
            v[j][1] = ldg_nc(xr + 2 * b + 1);
        }
    }
#pragma unroll
    for (int j = 0; j < RB; ++j)
        if (lane + 32 * j < nblk) add_sq(v[j][0], v[j][1]);
    for (int b = lane + 32 * RB; b < nblk; b += 32) add_sq(ldg_nc(xr + 2 * b), ldg_nc(xr + 2 * b + 1));
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) ss = __fadd_rn(ss, __shfl_xor_sync(0xFFFFFFFFu, ss, off));
    const float ms = __fdiv_rn(ss, static_cast<float>(K));
    const float inv = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(ms, eps)));

    // normalised values of one block: (x * inv) * g
    auto norm16 = [&](const uint4& a, const uint4& b, int blk, float (&n)[16]) {
        const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
        const float4* g4 = reinterpret_cast<const float4*>(g + 16 * blk);
        float gv[16];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float4 q = __ldg(g4 + i);
            gv[4 * i] = q.x;
            gv[4 * i + 1] = q.y;
            gv[4 * i + 2] = q.z;
            gv[4 * i + 3] = q.w;
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            n[2 * i] = __fmul_rn(__fmul_rn(__uint_as_float(w[i] << 16), inv), gv[2 * i]);
            n[2 * i + 1] = __fmul_rn(__fmul_rn(__uint_as_float(w[i] & 0xFFFF0000u), inv), gv[2 * i + 1]);
        }
    };
    // pass 2: absmax of the normalised values (bit patterns of |n| order like the values)
    uint32_t mx = 0;
    auto max16 = [&](const uint4& a, const uint4& b, int blk) {
        float n[16];
        norm16(a, b, blk, n);
#pragma unroll
        for (int i = 0; i < 16; ++i) mx = max(mx, __float_as_uint(n[i]) & 0x7FFFFFFFu);
    };
#pragma unroll
    for (int j = 0; j < RB; ++j)
        if (lane + 32 * j < nblk) max16(v[j][0], v[j][1], lane + 32 * j);
    for (int b = lane + 32 * RB; b < nblk; b += 32) max16(ldg_nc(xr + 2 * b), ldg_nc(xr + 2 * b + 1), b);
    mx = __reduce_max_sync(0xFFFFFFFFu, mx);
    bad = __reduce_or_sync(0xFFFFFFFFu, bad);
    if (lane == 0 && (bad || mx >= 0x7F800000u)) raise_status(status, kStatusNonfinite);
    const float s = __fdiv_rn(127.0f, fmaxf(__uint_as_float(mx), 1e-5f));
    if (lane == 0) s_tok[t] = s;

    // pass 3: quantise and store in the requested layout
    int8_t* out = xq + t * K;
    auto store16 = [&](const uint4& a, const uint4& b, int blk) {
        float n[16];
        norm16(a, b, blk, n);
        uint32_t q[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) q[i] = quant_code_bits(n[i], s);
        uint4 o;
        if (LAYOUT == kNatural)
            o = make_uint4(pack_codes(q[0], q[1], q[2], q[3]), pack_codes(q[4], q[5], q[6], q[7]),
                           pack_codes(q[8], q[9], q[10], q[11]), pack_codes(q[12], q[13], q[14], q[15]));
        else
            o = make_uint4(pack_codes(q[0], q[2], q[4], q[6]), pack_codes(q[1], q[3], q[5], q[7]),
                           pack_codes(q[8], q[10], q[12], q[14]), pack_codes(q[9], q[11], q[13], q[15]));
        *reinterpret_cast<uint4*>(out + 16 * static_cast<long long>(blk)) = o;
    };
#pragma unroll
    for (int j = 0; j < RB; ++j)
        if (lane + 32 * j < nblk) store16(v[j][0], v[j][1], lane + 32 * j);
    for (int b = lane + 32 * RB; b < nblk; b += 32) store16(ldg_nc(xr + 2 * b), ldg_nc(xr + 2 * b + 1), b);
}

// RMSNorm then per-token absmax int8 (layout as launch_quant); g fp32 [K]
// must be 16-byte aligned.
cudaError_t launch_rmsnorm_quant(const uint16_t* x, const float* g, float eps, long long T, long long K, int8_t* xq,
                                 float* s_tok, int layout, unsigned* status, cudaStream_t stream, void* zero16,
                                 long long nzero16) {
    const unsigned blocks = static_cast<unsigned>((T + 7) / 8);
    uint4* zw = static_cast<uint4*>(zero16);
    if (layout == kPairs)
        rmsnorm_quant_kernel<kPairs><<<blocks, 256, 0, stream>>>(x, g, eps, T, K, xq, s_tok, zw, nzero16, status);
    else
        rmsnorm_quant_kernel<kNatural><<<blocks, 256, 0, stream>>>(x, g, eps, T, K, xq, s_tok, zw, nzero16, status);
    return cudaGetLastError();
}

}  // namespace sbl
