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
// lanes (every lane ends with the same total).  Pass 1 loads up to RB of a
// lane's blocks at once (the rest in a loop); the absmax of the normalised
// values and the quantisation then read x again (from L1) in a coalesced
// mapping, which their order-free arithmetic allows.
// Non-finite input shows as a non-finite sum of squares (a square that
// overflows float32 does too) or normalised value, and sets the status bit.
// Pairs of floats in one 64-bit register, for the sm_100 paired float
// instructions (each half rounded exactly like the scalar IEEE operation).
__device__ __forceinline__ uint64_t f2(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ void f2split(uint64_t v, float& lo, float& hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t mul2(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ uint64_t add2(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
// Three-input max / min that propagate NaN.
__device__ __forceinline__ float max3n(float a, float b, float c) {
    float r;
    asm("max.NaN.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}
__device__ __forceinline__ float min3n(float a, float b, float c) {
    float r;
    asm("min.NaN.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

template <int LAYOUT, int RB>
__global__ void __launch_bounds__(256) rmsnorm_quant_kernel(const uint16_t* __restrict__ x,
                                                            const float* __restrict__ g, float eps, long long T,
                                                            long long K, int8_t* __restrict__ xq,
                                                            float* __restrict__ s_tok, uint4* __restrict__ zero_words,
                                                            long long nzero, unsigned* status) {
    asm volatile("griddepcontrol.launch_dependents;");
    zero_fill(zero_words, nzero);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long t = static_cast<long long>(blockIdx.x) * 8 + warp;
    if (t >= T) return;
    const uint4* xr = reinterpret_cast<const uint4*>(x + t * K);
    const int nblk = static_cast<int>(K >> 4);
    uint4 v[RB][2];
    // pass 1: sum of squares in the lane's k order
    float ss = 0.f;
    auto add_sq = [&](const uint4& a, const uint4& b) {
        const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const uint64_t p = f2(__uint_as_float(w[i] << 16), __uint_as_float(w[i] & 0xFFFF0000u));
            float lo, hi;
            f2split(mul2(p, p), lo, hi);  // squares of elements 2i and 2i + 1
            ss = __fadd_rn(ss, lo);
            ss = __fadd_rn(ss, hi);
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

    // Passes 2 and 3 take a coalesced mapping (any works: the absmax and the
    // elementwise quantisation do not depend on order): lane l handles the
    // four elements 4l + 128i .. 4l + 128i + 3, re-reading x (now in L1) with
    // 8-byte loads and g with 16-byte loads, every warp access contiguous.
    const uint64_t inv2 = f2(inv, inv);
    const uint2* xr2 = reinterpret_cast<const uint2*>(x + t * K);
    const float4* g4 = reinterpret_cast<const float4*>(g);
    const int nstripe = static_cast<int>((K + 127) >> 7);
    // (x * inv) * g of four elements, as two pairs
    auto norm4 = [&](int k4, uint64_t& n01, uint64_t& n23) {
        const uint2 w = __ldg(xr2 + k4);
        const float4 q = __ldg(g4 + k4);
        n01 = mul2(mul2(f2(__uint_as_float(w.x << 16), __uint_as_float(w.x & 0xFFFF0000u)), inv2), f2(q.x, q.y));
        n23 = mul2(mul2(f2(__uint_as_float(w.y << 16), __uint_as_float(w.y & 0xFFFF0000u)), inv2), f2(q.z, q.w));
    };
    // pass 2: largest and smallest normalised value (NaN propagates)
    float hi_v = 0.f, lo_v = 0.f;
    for (int i = 0; i < nstripe; ++i) {
        const int k4 = lane + 32 * i;  // index of the 4-element group
        if (4 * k4 < K) {
            uint64_t n01, n23;
            norm4(k4, n01, n23);
            float e0, e1, e2, e3;
            f2split(n01, e0, e1);
            f2split(n23, e2, e3);
            hi_v = max3n(hi_v, e0, e1);
            lo_v = min3n(lo_v, e0, e1);
            hi_v = max3n(hi_v, e2, e3);
            lo_v = min3n(lo_v, e2, e3);
        }
    }
    float amax = max3n(hi_v, -lo_v, 0.f);  // max |x_norm| of this lane (NaN if any value was NaN)
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) amax = max3n(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, off), 0.f);
    if (lane == 0 && !(fabsf(ss) <= 3.4028235e38f && amax <= 3.4028235e38f)) raise_status(status, kStatusNonfinite);
    const float s = __fdiv_rn(127.0f, fmaxf(amax, 1e-5f));
    if (lane == 0) s_tok[t] = s;

    // pass 3: quantise (quant_code_bits two at a time) and store.  In the
    // pairing layout a 16-element block's word q holds the even (q = 0, 2) or
    // odd (q = 1, 3) elements of lanes q & ~1 and q | 1, so neighbouring lanes
    // swap codes once and each stores the word at its own position.
    const uint64_t s2 = f2(s, s), magic2 = f2(12582912.0f, 12582912.0f);
    uint32_t* out = reinterpret_cast<uint32_t*>(xq + t * K);
    for (int i = 0; i < nstripe; ++i) {
        const int k4 = lane + 32 * i;
        const bool ok = 4 * k4 < K;  // whole 16-element blocks: lanes l and l ^ 1 agree
        uint32_t p = 0;
        if (ok) {
            uint64_t n01, n23;
            norm4(k4, n01, n23);
            float c0, c1, c2, c3;
            f2split(add2(mul2(n01, s2), magic2), c0, c1);
            f2split(add2(mul2(n23, s2), magic2), c2, c3);
            p = pack_codes(__float_as_uint(c0), __float_as_uint(c1), __float_as_uint(c2), __float_as_uint(c3));
        }
        if (LAYOUT == kNatural) {
            if (ok) out[k4] = p;
        } else {
            const uint32_t pp = __shfl_xor_sync(0xFFFFFFFFu, p, 1);
            const uint32_t word = (lane & 1) ? prmt(pp, p, 0x7531u) : prmt(p, pp, 0x6420u);
            if (ok) out[k4] = word;
        }
    }
}

template <int LAYOUT>
static void launch_rms_rb(const uint16_t* x, const float* g, float eps, long long T, long long K, int8_t* xq,
                          float* s_tok, uint4* zw, long long nzero, unsigned* status, cudaStream_t stream) {
    const unsigned blocks = static_cast<unsigned>((T + 7) / 8);
    const long long per_lane = ((K >> 4) + 31) / 32;  // blocks per lane
    if (per_lane <= 1)
        rmsnorm_quant_kernel<LAYOUT, 1><<<blocks, 256, 0, stream>>>(x, g, eps, T, K, xq, s_tok, zw, nzero, status);
    else if (per_lane <= 2)
        rmsnorm_quant_kernel<LAYOUT, 2><<<blocks, 256, 0, stream>>>(x, g, eps, T, K, xq, s_tok, zw, nzero, status);
    else
        rmsnorm_quant_kernel<LAYOUT, 4><<<blocks, 256, 0, stream>>>(x, g, eps, T, K, xq, s_tok, zw, nzero, status);
}

// RMSNorm then per-token absmax int8 (layout as launch_quant); g fp32 [K]
// must be 16-byte aligned.
cudaError_t launch_rmsnorm_quant(const uint16_t* x, const float* g, float eps, long long T, long long K, int8_t* xq,
                                 float* s_tok, int layout, unsigned* status, cudaStream_t stream, void* zero16,
                                 long long nzero16) {
    uint4* zw = static_cast<uint4*>(zero16);
    if (layout == kPairs)
        launch_rms_rb<kPairs>(x, g, eps, T, K, xq, s_tok, zw, nzero16, status, stream);
    else
        launch_rms_rb<kNatural>(x, g, eps, T, K, xq, s_tok, zw, nzero16, status, stream);
    return cudaGetLastError();
}

}  // namespace sbl
