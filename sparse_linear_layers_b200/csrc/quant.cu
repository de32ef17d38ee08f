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
// The kernel is itself a programmatic dependent (it waits for its predecessor
// before reading x) and signals its own dependents at entry: the contraction
// kernel that follows may start its prologue while this one runs.
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
    asm volatile("griddepcontrol.wait;" ::: "memory");  // the predecessor may write x or still read the slots
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
    asm volatile("griddepcontrol.wait;" ::: "memory");  // the predecessor may write x or still read the slots
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
    pdl_launch(quant_kernel<LAYOUT, TPT, BPT>, dim3(blocks), dim3(256), 0, stream, x, T, K, xq, s_tok, zero_words, nzero,
               status);
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
        pdl_launch(quant_kernel_loop<LAYOUT>, dim3(blocks), dim3(256), 0, stream, x, T, K, xq, s_tok, zero_words,
                   nzero, status);
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
// then the absmax quantisation above.  The sum of squares is the exact sum
// rounded once to float32 (no summation order changes it); every later step
// is one IEEE float32 operation.
// One warp per token; for the sum, lane l owns the 16-element blocks b with
// b % 32 == l (up to RB = 4 of them held in registers, the rest read again); the
// absmax of the normalised values and the quantisation then read x again
// (from L1) in a coalesced mapping, which their order-free arithmetic allows.
// Non-finite input, a sum of squares past the float32 range and a non-finite
// normalised value set the status bit.
//
// Exact sum of squares.  A finite bf16 value is x = M * 2^(E - 134), with
// E = max(biased exponent, 1) and M its 8-bit significand (implicit bit
// included; M < 128 for subnormals); x^2 = M^2 * 2^(2E - 268) exactly.  With
// E_max the token's largest E, n the elements a lane adds and
// w = floor((48 - ceil(log2 n)) / 2):
//  * window path: every x with E >= E_max - w times 2^c, c = w + 134 - E_max,
//    is an integer y < 2^(8 + w) (a power-of-two product, exact in float32);
//    y^2 < 2^(16 + 2w) is exact in float32 and converts exactly to a 64-bit
//    integer, and n of them stay below 2^64, so the lane's uint64 sum A is
//    exact.  Values with E_max - 2w <= E < E_max - w take the factor 2^(c + w)
//    into a second sum B under the same bound.  A * 2^(2w) + B is the lane's
//    sum as a 128-bit integer in units of 2^(-2c - 2w); the warp adds the
//    lanes' integers (below 2^114).
//  * limb path, for a token with a nonzero value below E_max - 2w or whose
//    factor 2^c or 2^(c + w) is not a float32 (all |x| below about 2^-80):
//    every square M^2 * 2^(2E - 2) (units of 2^-266) is added, as two 32-bit
//    halves, into eighteen 64-bit shared-memory columns of 32-bit limbs
//    (576 bits); the carries are resolved once at the end.
// The integer is rounded to 53 bits by round-to-odd (the last kept bit is set
// when any dropped bit is nonzero) and that double rounded to the nearest
// float32.  Rounding to odd with two or more extra bits, then to nearest,
// equals one rounding to nearest of the exact value (Boldo and Melquiond,
// "Emulation of FMA and correctly rounded sums: proved algorithms using
// rounding to odd", IEEE Trans. Computers 57(4), 2008); the float32 overflow
// threshold and subnormal spacing are representable at 53 bits, so both
// carry over.
constexpr int kSqLimbs = 18;

__device__ __forceinline__ double pow2d(int k) {  // 2^k for -1022 <= k <= 1023
    return __longlong_as_double(static_cast<long long>(1023 + k) << 52);
}

// The integer hi * 2^64 + lo, times 2^e0, rounded to 53 bits by round-to-odd.
__device__ __forceinline__ double u128_round_odd(uint64_t hi, uint64_t lo, int e0) {
    uint64_t m;
    int sh;  // weight of bit 0 of m, in bits of the integer
    if (hi == 0) {
        if ((lo >> 53) == 0) {
            m = lo;
            sh = 0;
        } else {
            const int lz = __clzll(static_cast<long long>(lo));  // at most 10
            const uint64_t top = lo << lz;
            m = (top >> 11) | ((top & 0x7FFull) != 0 ? 1ull : 0ull);
            sh = 11 - lz;
        }
    } else {
        const int lz = __clzll(static_cast<long long>(hi));
        const uint64_t top = lz ? (hi << lz) | (lo >> (64 - lz)) : hi;
        const uint64_t rest = lz ? (lo << lz) : lo;
        m = (top >> 11) | (((top & 0x7FFull) | rest) != 0 ? 1ull : 0ull);
        sh = 75 - lz;
    }
    return __ull2double_rn(m) * pow2d(e0 + sh);  // m < 2^53: both exact
}

// Resolve the carries of the limb columns (32-bit limbs in 64-bit words,
// units of 2^-266) and round the integer to 53 bits by round-to-odd.
__device__ double limbs_round_odd(const unsigned long long* col) {
    uint32_t w[kSqLimbs];
    unsigned long long carry = 0;
#pragma unroll
    for (int i = 0; i < kSqLimbs; ++i) {
        const unsigned long long t = col[i] + carry;
        w[i] = static_cast<uint32_t>(t);
        carry = t >> 32;
    }
    int h = 3;
    for (int i = kSqLimbs - 1; i > 3; --i)
        if (w[i] != 0u) {
            h = i;
            break;
        }
    uint32_t sticky = 0;
    for (int i = 0; i < h - 3; ++i) sticky |= w[i];
    const uint64_t hi = (static_cast<uint64_t>(w[h]) << 32) | w[h - 1];
    const uint64_t lo = ((static_cast<uint64_t>(w[h - 2]) << 32) | w[h - 3]) | (sticky ? 1ull : 0ull);
    return u128_round_odd(hi, lo, -266 + 32 * (h - 3));
}

__device__ __forceinline__ void add128(uint64_t& hi, uint64_t& lo, uint64_t bhi, uint64_t blo) {
    asm("add.cc.u64 %0, %0, %2;\n\taddc.u64 %1, %1, %3;" : "+l"(lo), "+l"(hi) : "l"(blo), "l"(bhi));
}

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
    asm volatile("griddepcontrol.wait;" ::: "memory");  // the predecessor may write x or still read the slots
    zero_fill(zero_words, nzero);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long t = static_cast<long long>(blockIdx.x) * 8 + warp;
    if (t >= T) return;
    const uint4* xr = reinterpret_cast<const uint4*>(x + t * K);
    const int nblk = static_cast<int>(K >> 4);
    uint4 v[RB][2];
#pragma unroll
    for (int j = 0; j < RB; ++j) {
        const int b = lane + 32 * j;
        if (b < nblk) {
            v[j][0] = ldg_nc(xr + 2 * b);
            v[j][1] = ldg_nc(xr + 2 * b + 1);
        } else {
            v[j][0] = v[j][1] = make_uint4(0u, 0u, 0u, 0u);
        }
    }
    // Apply f to every 32-bit word (two bf16 values) of the lane's blocks.
    auto each_word = [&](auto&& f) {
#pragma unroll
        for (int j = 0; j < RB; ++j) {
            f(v[j][0].x); f(v[j][0].y); f(v[j][0].z); f(v[j][0].w);
            f(v[j][1].x); f(v[j][1].y); f(v[j][1].z); f(v[j][1].w);
        }
        for (int b = lane + 32 * RB; b < nblk; b += 32) {
            const uint4 a0 = ldg_nc(xr + 2 * b), a1 = ldg_nc(xr + 2 * b + 1);
            f(a0.x); f(a0.y); f(a0.z); f(a0.w);
            f(a1.x); f(a1.y); f(a1.z); f(a1.w);
        }
    };
    // pass 0: largest magnitude and smallest nonzero magnitude (bf16 bits;
    // the halves of a word are handled as 16-bit lanes, a zero maps to 0xFFFF)
    uint32_t mx2 = 0, mn2 = 0xFFFFFFFFu;
    each_word([&](uint32_t w) {
        const uint32_t m2 = w & 0x7FFF7FFFu;
        mx2 = __vmaxu2(mx2, m2);
        mn2 = __vminu2(mn2, (m2 + 0x7FFF7FFFu) ^ 0x80008000u);  // per half: mag - 1, or 0xFFFF for 0
    });
    const uint32_t mx = __reduce_max_sync(0xFFFFFFFFu, max(mx2 & 0xFFFFu, mx2 >> 16));
    const uint32_t mn = __reduce_min_sync(0xFFFFFFFFu, min(mn2 & 0xFFFFu, mn2 >> 16)) + 1u;

    // pass 1: the exact sum of squares, rounded once to float32
    float ss;
    if (mx >= 0x7F80u) {
        ss = __int_as_float(0x7FC00000);  // Inf or NaN in x
    } else if (mx == 0u) {
        ss = 0.f;
    } else {
        const int e_max = max(static_cast<int>(mx >> 7), 1), e_min = max(static_cast<int>(mn >> 7), 1);
        const int per_lane = 16 * ((nblk + 31) >> 5);
        const int win = (48 - (32 - __clz(per_lane - 1))) >> 1;
        const int c = win + 134 - e_max;
        uint64_t hi = 0, lo = 0;
        int e0 = 0;
        const bool one_window = e_max - e_min <= win && c <= 127;
        const bool two_windows = !one_window && e_max - e_min <= 2 * win && c + win <= 127;
        if (one_window) {
            const float fc = __uint_as_float(static_cast<uint32_t>(127 + c) << 23);  // 2^c
            const uint64_t c2 = f2(fc, fc);
            uint64_t acc = 0;
            each_word([&](uint32_t w) {
                uint64_t y = mul2(f2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u)), c2);
                float q0, q1;
                f2split(mul2(y, y), q0, q1);
                acc += __float2ull_rz(q0) + __float2ull_rz(q1);
            });
            lo = acc;
            e0 = -2 * c;
        } else if (two_windows) {
            const float fa = __uint_as_float(static_cast<uint32_t>(127 + c) << 23);        // 2^c
            const float fb = __uint_as_float(static_cast<uint32_t>(127 + c + win) << 23);  // 2^(c + w)
            const uint32_t thr = static_cast<uint32_t>(e_max - win) << 7;  // E >= E_max - w (here E_max - w >= 2)
            uint64_t acc_a = 0, acc_b = 0;
            each_word([&](uint32_t w) {
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const uint32_t bits = h ? (w & 0xFFFF0000u) : (w << 16);
                    const bool big = ((bits >> 16) & 0x7FFFu) >= thr;
                    const float y = __fmul_rn(__uint_as_float(bits), big ? fa : fb);
                    const uint64_t q = __float2ull_rz(__fmul_rn(y, y));
                    acc_a += big ? q : 0ull;
                    acc_b += big ? 0ull : q;
                }
            });
            hi = acc_a >> (64 - 2 * win);
            lo = acc_a << (2 * win);
            add128(hi, lo, 0ull, acc_b);
            e0 = -2 * c - 2 * win;
        }
        if (one_window || two_windows) {
#pragma unroll
            for (int off = 16; off >= 1; off >>= 1)
                add128(hi, lo, __shfl_xor_sync(0xFFFFFFFFu, hi, off), __shfl_xor_sync(0xFFFFFFFFu, lo, off));
            ss = __double2float_rn(u128_round_odd(hi, lo, e0));
        } else {
            __shared__ unsigned long long sq_limbs[8][kSqLimbs];
            unsigned long long* col = sq_limbs[warp];
            if (lane < kSqLimbs) col[lane] = 0ull;
            __syncwarp();
            each_word([&](uint32_t w) {
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const uint32_t mag = (h ? (w >> 16) : w) & 0x7FFFu;
                    if (mag != 0u) {
                        const uint32_t e = mag >> 7;
                        const uint32_t M = e ? ((mag & 0x7Fu) | 0x80u) : mag;
                        const uint32_t p = 2u * max(e, 1u) - 2u;  // M^2 * 2^p in units of 2^-266
                        const unsigned long long t = static_cast<unsigned long long>(M * M) << (p & 31u);
                        atomicAdd(col + (p >> 5), t & 0xFFFFFFFFull);
                        atomicAdd(col + (p >> 5) + 1, t >> 32);
                    }
                }
            });
            __syncwarp();
            float s0 = 0.f;
            if (lane == 0) s0 = __double2float_rn(limbs_round_odd(col));
            ss = __shfl_sync(0xFFFFFFFFu, s0, 0);
        }
    }
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
    // The product x_norm * s and the rounding add are scalar IEEE operations
    // (quant_code_bits): a paired multiply followed by a paired add was
    // observed to round like one fused multiply-add, which decides ties of
    // x_norm * s (exactly k + 1/2 after rounding, not before) the wrong way.
    uint32_t* out = reinterpret_cast<uint32_t*>(xq + t * K);
    for (int i = 0; i < nstripe; ++i) {
        const int k4 = lane + 32 * i;
        const bool ok = 4 * k4 < K;  // whole 16-element blocks: lanes l and l ^ 1 agree
        uint32_t p = 0;
        if (ok) {
            uint64_t n01, n23;
            norm4(k4, n01, n23);
            float c0, c1, c2, c3;
            f2split(n01, c0, c1);
            f2split(n23, c2, c3);
            p = pack_codes(quant_code_bits(c0, s), quant_code_bits(c1, s), quant_code_bits(c2, s),
                           quant_code_bits(c3, s));
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
    // blocks per lane held in registers: up to four (rows up to K = 2048); the
    // rest of a longer row is read again from L1/L2 in each pass.  Holding whole
    // rows of K = 4864 (ten blocks, 128 registers) cut the resident warps from
    // about 54% to 21% and ran slower (ncu), so four is the limit.
    const long long per_lane = ((K >> 4) + 31) / 32;
    if (per_lane <= 1)
        pdl_launch(rmsnorm_quant_kernel<LAYOUT, 1>, dim3(blocks), dim3(256), 0, stream, x, g, eps, T, K, xq, s_tok, zw, nzero, status);
    else if (per_lane <= 2)
        pdl_launch(rmsnorm_quant_kernel<LAYOUT, 2>, dim3(blocks), dim3(256), 0, stream, x, g, eps, T, K, xq, s_tok, zw, nzero, status);
    else
        pdl_launch(rmsnorm_quant_kernel<LAYOUT, 4>, dim3(blocks), dim3(256), 0, stream, x, g, eps, T, K, xq, s_tok, zw, nzero, status);
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
