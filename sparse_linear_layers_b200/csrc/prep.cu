// Weight preparation: N:M magnitude mask, per-row absmean scale over the kept
// weights, ternarisation and 2-bit packing, fused in one pass per row.
//
// Operator: Sparse-BitNet Guide: 1.58-Bit LLMs Meet 2:4 Sparsity, "Mathematical
// Formulation of Sparse-BitLinear" (mask equation, joint sparse-ternary
// equation); per-row absmean from the halo-sparse-bitnet-3:4-500m card,
// "Recipe"; code table 00 = 0, 01 = +1, 10 = -1 from its "Packed vs raw".
//
// One to eight warps share a row; each thread owns up to two 16-weight chunks,
// read once as 16-byte loads and kept in registers.  Pass 1 applies the N:M
// mask to the registers and finds the row's largest and smallest kept
// magnitudes, pass 2 adds the kept |w| exactly (see kWin), pass 3 ternarises
// the registers against the row scale and writes one 32-bit word of codes
// (and optionally 16 mask bits) per chunk.  Rows longer than 512 chunks
// (K > 8192) use a warp-per-row variant that reads the row twice and sums in
// shared-memory limbs.
//
// Exact sum: a finite float |w| = m * 2^(p - 149) with a 24-bit integer m and
// 0 <= p <= 253, so the row sum is an integer in units of 2^-149 below 2^300.
// Each lane keeps it in ten 32-bit limbs held in 64-bit shared-memory words
// (carries are resolved once, at the end), which makes the sum independent of
// the order of additions; the total is rounded once to double.
#include "sbl_common.cuh"

namespace sbl {

constexpr int kPrepWarps = 8;
constexpr int kLimbs = 10;

__device__ __forceinline__ void exact_add(unsigned long long* limb_col, uint32_t abs_bits) {
    const uint32_t e = abs_bits >> 23;
    const uint32_t m24 = (abs_bits & 0x7FFFFFu) | (e ? 0x800000u : 0u);
    const uint32_t p = e ? e - 1u : 0u;
    const uint32_t li = p >> 5;
    const unsigned long long v = static_cast<unsigned long long>(m24) << (p & 31u);
    limb_col[li * 32] += v & 0xFFFFFFFFull;
    limb_col[(li + 1) * 32] += v >> 32;
}

// Round the 320-bit integer w[0..9] (32-bit limbs, units of 2^-149) to double.
__device__ double limbs_to_double(const uint32_t (&w)[kLimbs]) {
    int h = -1;
#pragma unroll
    for (int i = kLimbs - 1; i >= 0; --i)
        if (h < 0 && w[i] != 0u) h = i;
    const double two_m149 = 1.4012984643248170709e-45;  // 2^-149, exact
    if (h < 0) return 0.0;
    if (h <= 1) {
        const unsigned long long x = (static_cast<unsigned long long>(w[1]) << 32) | w[0];
        return __ull2double_rn(x) * two_m149;
    }
    const int lz = __clz(w[h]);
    unsigned long long top;
    uint32_t dropped;
    if (lz == 0) {
        top = (static_cast<unsigned long long>(w[h]) << 32) | w[h - 1];
        dropped = w[h - 2];
    } else {
        top = (static_cast<unsigned long long>(w[h]) << (32 + lz)) |
              (static_cast<unsigned long long>(w[h - 1]) << lz) | (w[h - 2] >> (32 - lz));
        dropped = w[h - 2] & ((1u << (32 - lz)) - 1u);
    }
    for (int i = 0; i < h - 2; ++i) dropped |= w[i];
    top |= (dropped != 0u) ? 1ull : 0ull;  // sticky bit: below the rounding position
    const int e2 = 32 * h - 32 - lz - 149;  // weight of bit 0 of `top`
    const double scale = __longlong_as_double(static_cast<long long>(1023 + e2) << 52);
    return __ull2double_rn(top) * scale;
}

// keep[i] for the M weights of one group: rank by magnitude, ties to the lower index.
template <int M>
__device__ __forceinline__ uint32_t group_keep_bits(const uint32_t* a, int n) {
    int rank[M];
#pragma unroll
    for (int j = 0; j < M; ++j) rank[j] = 0;
#pragma unroll
    for (int i = 0; i < M; ++i)
#pragma unroll
        for (int j = i + 1; j < M; ++j) {
            if (a[i] >= a[j]) ++rank[j];
            else ++rank[i];
        }
    uint32_t bits = 0;
#pragma unroll
    for (int j = 0; j < M; ++j) bits |= (rank[j] < n ? 1u : 0u) << j;
    return bits;
}

template <int M>
__device__ __forceinline__ uint32_t chunk_keep_bits(const uint32_t (&a)[16], int n) {
    uint32_t bits = 0;
#pragma unroll
    for (int g = 0; g < 16 / M; ++g) bits |= group_keep_bits<M>(a + g * M, n) << (g * M);
    return bits;
}

__device__ __forceinline__ void load_chunk(const float* p, uint32_t (&bits)[16]) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const uint4 v = ldg_nc(p + 4 * q);
        bits[4 * q + 0] = v.x;
        bits[4 * q + 1] = v.y;
        bits[4 * q + 2] = v.z;
        bits[4 * q + 3] = v.w;
    }
}

// The scale as the halo card stores it ("Packed vs raw": one bf16 row_scale per
// row): round to nearest even bf16 when asked, before it ternarises the row.
__device__ __forceinline__ float scale_storage(float sc, int scale_bf16) {
    return scale_bf16 ? __bfloat162float(__float2bfloat16_rn(sc)) : sc;
}

template <int M>
__global__ void __launch_bounds__(kPrepWarps * 32) prep_kernel(const float* __restrict__ W, long long O, long long K,
                                                               int n, uint8_t* __restrict__ packed,
                                                               float* __restrict__ row_scale,
                                                               uint8_t* __restrict__ mask_bits, int scale_bf16,
                                                               const float* __restrict__ ext_scale, unsigned* status) {
    __shared__ unsigned long long limbs[kPrepWarps][kLimbs][32];
    __shared__ unsigned long long totals[kPrepWarps][kLimbs];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long row = static_cast<long long>(blockIdx.x) * kPrepWarps + warp;
    if (row >= O) return;  // whole warps leave together; no block barrier below

    const float* wr = W + row * K;
    const int nchunks = static_cast<int>(K >> 4);
    unsigned long long* my = &limbs[warp][0][lane];
#pragma unroll
    for (int l = 0; l < kLimbs; ++l) my[l * 32] = 0ull;

    bool bad = false;
    for (int c = lane; c < nchunks; c += 32) {
        uint32_t a[16];
        load_chunk(wr + 16 * c, a);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            a[i] &= 0x7FFFFFFFu;
            bad |= a[i] >= 0x7F800000u;
        }
        const uint32_t keep = chunk_keep_bits<M>(a, n);
#pragma unroll
        for (int i = 0; i < 16; ++i)
            if (keep & (1u << i)) exact_add(my, a[i]);
    }
    __syncwarp();
    if (lane < kLimbs) {
        unsigned long long s = 0;
        for (int i = 0; i < 32; ++i) s += limbs[warp][lane][i];
        totals[warp][lane] = s;
    }
    __syncwarp();

    float scale = 0.f;
    if (lane == 0) {
        uint32_t w[kLimbs];
        unsigned long long carry = 0;
#pragma unroll
        for (int i = 0; i < kLimbs; ++i) {
            const unsigned long long t = totals[warp][i] + carry;
            w[i] = static_cast<uint32_t>(t);
            carry = t >> 32;
        }
        const double sum = limbs_to_double(w);
        const double kept = static_cast<double>((K / M) * n);
        scale = ext_scale ? *ext_scale : scale_storage(fmaxf(__double2float_rn(__ddiv_rn(sum, kept)), 1e-5f), scale_bf16);
        row_scale[row] = scale;
    }
    scale = __shfl_sync(0xFFFFFFFFu, scale, 0);
    if (__any_sync(0xFFFFFFFFu, bad) && lane == 0) raise_status(status, kStatusNonfinite);

    const uint32_t half_bits = __float_as_uint(0.5f * scale);  // exact: scale >= 1e-5 is normal
    uint32_t* prow = reinterpret_cast<uint32_t*>(packed + row * (K >> 2));
    uint16_t* mrow = mask_bits ? reinterpret_cast<uint16_t*>(mask_bits + row * (K >> 3)) : nullptr;
    for (int c = lane; c < nchunks; c += 32) {
        uint32_t raw[16], a[16];
        load_chunk(wr + 16 * c, raw);
#pragma unroll
        for (int i = 0; i < 16; ++i) a[i] = raw[i] & 0x7FFFFFFFu;
        const uint32_t keep = chunk_keep_bits<M>(a, n);
        uint32_t codes = 0;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            // round(w / scale) != 0  <=>  |w| / scale > 1/2  <=>  |w| > scale / 2 (exact compare)
            const bool nz = ((keep >> i) & 1u) && (a[i] > half_bits);
            const uint32_t code = nz ? ((raw[i] >> 31) ? 2u : 1u) : 0u;
            codes |= code << (2 * i);
        }
        prow[c] = codes;
        if (mrow) mrow[c] = static_cast<uint16_t>(keep);
    }
}

// ---------------------------------------------------------------------------
// Register-resident variant: each thread owns two 16-weight chunks of a row,
// WPR warps share a row and a block holds 8 / WPR rows.
//
// Exact row sum.  A finite float is |w| = m * 2^(e - 150) with e its biased
// exponent field (normal values; m < 2^24).  With e_max that of the row's
// largest magnitude and e_b = e_max - kWin, every kept value with e >= e_b is
// an integer below 2^(24 + kWin) in units of 2^(e_b - 150); a thread adds at
// most 32 of them, so the sum stays below 2^53 and accumulates in a double
// without rounding (one fused multiply-add by the power of two 2^(150 - e_b)
// per weight).  Thread sums are then added as 64-bit integers.  When
// e_b <= 0 every value of the row, subnormals included, is such an integer.
// A row in which a kept nonzero magnitude lies below 2^(e_b - 127) is summed
// instead with exact 320-bit shared-memory limbs; which rows do is known from
// the row minimum before any summing.
constexpr int kWin = 24;
constexpr int kChunksPerThread = 2;

// Bit 31 is set exactly when a >= b (both below 2^31).
__device__ __forceinline__ uint32_t ge_bit(uint32_t a, uint32_t b) { return b - a - 1u; }

// Drop flags (bit 31) of one group of four magnitudes, ties going to the lower
// index: a weight is dropped when it loses to at least N of the other three
// (N = 3: to all three; N = 2: to two or more).
template <int N>
__device__ __forceinline__ void drop4(const uint32_t* a, uint32_t (&d)[4]) {
    const uint32_t g01 = ge_bit(a[0], a[1]), g02 = ge_bit(a[0], a[2]), g03 = ge_bit(a[0], a[3]);
    const uint32_t g12 = ge_bit(a[1], a[2]), g13 = ge_bit(a[1], a[3]), g23 = ge_bit(a[2], a[3]);
    // losses: 0 loses to k when !g0k; 1 loses to 0 when g01, to k > 1 when !g1k; ...
    if constexpr (N == 3) {
        d[0] = ~g01 & ~g02 & ~g03;
        d[1] = g01 & ~g12 & ~g13;
        d[2] = g02 & g12 & ~g23;
        d[3] = g03 & g13 & g23;
    } else {
        d[0] = (~g01 & ~g02) | (~g01 & ~g03) | (~g02 & ~g03);
        d[1] = (g01 & ~g12) | (g01 & ~g13) | (~g12 & ~g13);
        d[2] = (g02 & g12) | (g02 & ~g23) | (g12 & ~g23);
        d[3] = (g03 & g13) | (g03 & g23) | (g13 & g23);
    }
}

template <int WPR>
__device__ __forceinline__ void row_sync() {
    if constexpr (WPR == 1) __syncwarp();
    else __syncthreads();
}

// The matrices of one launch (equal K), their rows stacked: matrix g owns the
// rows row_end[g - 1] .. row_end[g] - 1 of the launch.  A single matrix is G = 1.
constexpr int kPrepMaxGroup = 8;
struct PrepGroup {
    const float* W[kPrepMaxGroup];
    uint8_t* packed[kPrepMaxGroup];
    float* row_scale[kPrepMaxGroup];
    uint8_t* mask_bits[kPrepMaxGroup];
    long long row_end[kPrepMaxGroup];
    int G;
};

template <int M, int N, int WPR, bool WITH_MASK>
__global__ void __launch_bounds__((8 / WPR) * WPR * 32) prep_kernel_rr(const PrepGroup grp, long long K,
                                                                      int scale_bf16, const float* __restrict__ ext_scale,
                                                                      unsigned* status) {
    constexpr int RPB = 8 / WPR;  // rows per block
    constexpr int TPR = WPR * 32;
    constexpr int CPT = kChunksPerThread;
    __shared__ uint32_t wmax[RPB * WPR], wmin[RPB * WPR];
    __shared__ unsigned long long wsum[RPB * WPR];
    __shared__ unsigned long long limbs[RPB][kLimbs];
    __shared__ float scales[RPB];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int sub = threadIdx.x / TPR, tr = threadIdx.x % TPR;
    const long long grow = static_cast<long long>(blockIdx.x) * RPB + sub;  // row of the stacked matrices
    const bool valid = grow < grp.row_end[grp.G - 1];
    // the matrix of this row (constant indices only)
    const float* W = grp.W[0];
    uint8_t* packed = grp.packed[0];
    float* row_scale = grp.row_scale[0];
    uint8_t* mask_bits = grp.mask_bits[0];
    long long row = grow;
    if (grp.G > 1)
#pragma unroll
        for (int i = 1; i < kPrepMaxGroup; ++i)
            if (i < grp.G && grow >= grp.row_end[i - 1]) {
                W = grp.W[i];
                packed = grp.packed[i];
                row_scale = grp.row_scale[i];
                mask_bits = grp.mask_bits[i];
                row = grow - grp.row_end[i - 1];
            }
    const int nchunks = static_cast<int>(K >> 4);
    const float* wr = W + (valid ? row : 0) * K;

    // kr: the weight's bits when it is kept, 0 when it is dropped
    uint32_t kr[CPT][16];
#pragma unroll
    for (int j = 0; j < CPT; ++j) {
        const int c = tr + TPR * j;
        if (valid && c < nchunks) load_chunk(wr + 16 * c, kr[j]);
        else
#pragma unroll
            for (int i = 0; i < 16; ++i) kr[j][i] = 0u;
    }

    // pass 1: N:M mask, row maximum of |w|, row minimum of the kept nonzero |w|
    uint32_t mx = 0, mn2 = 0xFFFFFFFFu, kbits = 0;
#pragma unroll
    for (int j = 0; j < CPT; ++j) {
        if constexpr (M == 4) {
#pragma unroll
            for (int g = 0; g < 4; ++g) {
                uint32_t a[4], d[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) a[q] = kr[j][4 * g + q] & 0x7FFFFFFFu;
                mx = __vimax3_u32(mx, a[0], a[1]);
                mx = __vimax3_u32(mx, a[2], a[3]);
                drop4<N>(a, d);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    kr[j][4 * g + q] &= ~static_cast<uint32_t>(static_cast<int>(d[q]) >> 31);
                    if constexpr (WITH_MASK) kbits |= ((~d[q]) >> 31) << (16 * j + 4 * g + q);
                }
            }
        } else {
            uint32_t a[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) a[i] = kr[j][i] & 0x7FFFFFFFu;
#pragma unroll
            for (int i = 0; i < 16; i += 2) mx = __vimax3_u32(mx, a[i], a[i + 1]);
            const uint32_t keep = group_keep_bits<8>(a, N) | (group_keep_bits<8>(a + 8, N) << 8);
#pragma unroll
            for (int i = 0; i < 16; ++i) kr[j][i] = ((keep >> i) & 1u) ? kr[j][i] : 0u;
            if constexpr (WITH_MASK) kbits |= keep << (16 * j);
        }
        // 2|w| - 1 over the kept weights: zeros wrap to the largest value
#pragma unroll
        for (int i = 0; i < 16; i += 2) mn2 = __vimin3_u32(mn2, (kr[j][i] << 1) - 1u, (kr[j][i + 1] << 1) - 1u);
    }
    mx = __reduce_max_sync(0xFFFFFFFFu, mx);
    mn2 = __reduce_min_sync(0xFFFFFFFFu, mn2);
    if constexpr (WPR > 1) {
        if (lane == 0) {
            wmax[warp] = mx;
            wmin[warp] = mn2;
        }
        __syncthreads();
#pragma unroll
        for (int w = 0; w < WPR; ++w) {
            mx = max(mx, wmax[sub * WPR + w]);
            mn2 = min(mn2, wmin[sub * WPR + w]);
        }
    }
    if (mx >= 0x7F800000u && tr == 0 && valid) raise_status(status, kStatusNonfinite);
    const int emax = static_cast<int>(mx >> 23);
    const int eb = emax - kWin;
    // a kept nonzero magnitude below 2^(eb - 127) leaves the window
    const bool exact_path = eb >= 1 && mn2 < (static_cast<uint32_t>(eb) << 24) - 1u;

    // pass 2: the sum of the kept |w|
    double sum;
    bool any_exact;
    if constexpr (WPR == 1) any_exact = exact_path;  // warp-uniform
    else any_exact = __syncthreads_or(exact_path);
    if (!exact_path) {
        const double up = __longlong_as_double(static_cast<long long>(1023 + 150 - eb) << 52);  // 2^(150 - eb)
        double acc = 0.0;
#pragma unroll
        for (int j = 0; j < CPT; ++j)
#pragma unroll
            for (int i = 0; i < 16; ++i) acc = fma(static_cast<double>(fabsf(__uint_as_float(kr[j][i]))), up, acc);
        unsigned long long t = __double2ull_rn(acc);  // an integer below 2^53
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) t += __shfl_xor_sync(0xFFFFFFFFu, t, off);
        if constexpr (WPR > 1) {
            if (lane == 0) wsum[warp] = t;
        } else {
            // units of 2^(eb - 150); the row total is below 2^61
            sum = __ull2double_rn(t) * __longlong_as_double(static_cast<long long>(1023 + eb - 150) << 52);
        }
    }
    if (any_exact) {
        // exact 320-bit limbs (units of 2^-149), integer adds in any order
        if (tr < kLimbs) limbs[sub][tr] = 0ull;
        row_sync<WPR>();
        if (exact_path) {
#pragma unroll
            for (int j = 0; j < CPT; ++j)
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const uint32_t a = kr[j][i] & 0x7FFFFFFFu;
                    if (a == 0u) continue;
                    const uint32_t e = a >> 23;
                    const uint32_t m24 = (a & 0x7FFFFFu) | (e ? 0x800000u : 0u);
                    const uint32_t p = e ? e - 1u : 0u;
                    const unsigned long long v = static_cast<unsigned long long>(m24) << (p & 31u);
                    atomicAdd(&limbs[sub][p >> 5], v & 0xFFFFFFFFull);
                    atomicAdd(&limbs[sub][(p >> 5) + 1], v >> 32);
                }
        }
        row_sync<WPR>();
        if (exact_path && (WPR == 1 || tr == 0)) {
            uint32_t w32[kLimbs];
            unsigned long long carry = 0;
#pragma unroll
            for (int i = 0; i < kLimbs; ++i) {
                const unsigned long long v = limbs[sub][i] + carry;
                w32[i] = static_cast<uint32_t>(v);
                carry = v >> 32;
            }
            sum = limbs_to_double(w32);
        }
    } else if constexpr (WPR > 1) {
        __syncthreads();
    }
    float sc;
    const double kept = static_cast<double>((K / M) * N);
    if constexpr (WPR > 1) {
        if (tr == 0) {
            if (!exact_path) {
                unsigned long long tot = 0;
#pragma unroll
                for (int w = 0; w < WPR; ++w) tot += wsum[sub * WPR + w];
                sum = __ull2double_rn(tot) * __longlong_as_double(static_cast<long long>(1023 + eb - 150) << 52);
            }
            sc = ext_scale ? *ext_scale : scale_storage(fmaxf(__double2float_rn(__ddiv_rn(sum, kept)), 1e-5f), scale_bf16);
            scales[sub] = sc;
            if (valid) row_scale[row] = sc;
        }
        __syncthreads();
        sc = scales[sub];
    } else {
        sc = ext_scale ? *ext_scale : scale_storage(fmaxf(__double2float_rn(__ddiv_rn(sum, kept)), 1e-5f), scale_bf16);
        if (lane == 0 && valid) row_scale[row] = sc;
    }
    if (!valid) return;

    // pass 3: ternarise and pack.  round(w / scale) != 0 exactly when
    // |w| > scale / 2, an exact compare (scale >= 1e-5 is normal, so halving
    // it is exact); the code is 01 for +1 and 10 for -1.  With s the sign bit
    // and a = |w| (both below 2^31), bit 31 of half - (s * 2^31 + a) is
    // (a > half) XOR s.  Two funnel shifts per weight stack s at bit 2i + 1
    // and that bit at bit 2i (weights 15 down to 0); then +1 = x AND NOT s
    // and -1 = s AND NOT x.  A dropped weight is 0 here, so x = s = 0.
    const uint32_t half_bits = __float_as_uint(0.5f * sc);
    uint32_t* prow = reinterpret_cast<uint32_t*>(packed + row * (K >> 2));
    uint16_t* mrow = (WITH_MASK && mask_bits) ? reinterpret_cast<uint16_t*>(mask_bits + row * (K >> 3)) : nullptr;
#pragma unroll
    for (int j = 0; j < CPT; ++j) {
        const int c = tr + TPR * j;
        if (c >= nchunks) continue;
        uint32_t acc = 0;
#pragma unroll
        for (int i = 15; i >= 0; --i) {
            acc = __funnelshift_l(kr[j][i], acc, 1);                   // s
            acc = __funnelshift_l(half_bits - kr[j][i], acc, 1);  // (|w| > scale / 2) XOR s
        }
        prow[c] = (acc & ~(acc >> 1) & 0x55555555u) | (acc & ~(acc << 1) & 0xAAAAAAAAu);
        if constexpr (WITH_MASK)
            if (mrow) mrow[c] = static_cast<uint16_t>(kbits >> (16 * j));
    }
}

template <int M, int N, int WPR>
static void launch_prep_rr(const PrepGroup& grp, long long K, bool with_mask, int scale_bf16, const float* ext_scale,
                           unsigned* status, cudaStream_t stream) {
    constexpr int RPB = 8 / WPR;
    const unsigned blocks = static_cast<unsigned>((grp.row_end[grp.G - 1] + RPB - 1) / RPB);
    if (with_mask)
        prep_kernel_rr<M, N, WPR, true><<<blocks, RPB * WPR * 32, 0, stream>>>(grp, K, scale_bf16, ext_scale, status);
    else
        prep_kernel_rr<M, N, WPR, false><<<blocks, RPB * WPR * 32, 0, stream>>>(grp, K, scale_bf16, ext_scale, status);
}

// Warps per row: the fewest that give every 16-weight chunk a slot (0: the
// row is longer than eight warps hold, K > 8192).
static int prep_wpr(long long K) {
    const long long wpr = ((K >> 4) + 32 * kChunksPerThread - 1) / (32 * kChunksPerThread);
    return wpr <= 8 ? static_cast<int>(wpr) : 0;
}

template <int M, int N>
static void launch_prep_group(const PrepGroup& grp, long long K, bool with_mask, int scale_bf16,
                              const float* ext_scale, unsigned* status, cudaStream_t stream) {
    switch (prep_wpr(K)) {
        case 1: launch_prep_rr<M, N, 1>(grp, K, with_mask, scale_bf16, ext_scale, status, stream); break;
        case 2: launch_prep_rr<M, N, 2>(grp, K, with_mask, scale_bf16, ext_scale, status, stream); break;
        case 3: launch_prep_rr<M, N, 3>(grp, K, with_mask, scale_bf16, ext_scale, status, stream); break;
        case 4: launch_prep_rr<M, N, 4>(grp, K, with_mask, scale_bf16, ext_scale, status, stream); break;
        case 5: launch_prep_rr<M, N, 5>(grp, K, with_mask, scale_bf16, ext_scale, status, stream); break;
        case 6: launch_prep_rr<M, N, 6>(grp, K, with_mask, scale_bf16, ext_scale, status, stream); break;
        case 7: launch_prep_rr<M, N, 7>(grp, K, with_mask, scale_bf16, ext_scale, status, stream); break;
        case 8: launch_prep_rr<M, N, 8>(grp, K, with_mask, scale_bf16, ext_scale, status, stream); break;
        default:  // rows longer than the register-resident kernel holds: one launch per matrix
            for (int g = 0; g < grp.G; ++g) {
                const long long O = grp.row_end[g] - (g ? grp.row_end[g - 1] : 0);
                if (O == 0) continue;
                const unsigned blocks = static_cast<unsigned>((O + kPrepWarps - 1) / kPrepWarps);
                prep_kernel<M><<<blocks, kPrepWarps * 32, 0, stream>>>(grp.W[g], O, K, N, grp.packed[g],
                                                                       grp.row_scale[g], grp.mask_bits[g],
                                                                       scale_bf16, ext_scale, status);
            }
    }
}

template <int M, int N>
static void launch_prep_mn(const float* W, long long O, long long K, uint8_t* packed, float* row_scale,
                           uint8_t* mask_bits, int scale_bf16, const float* ext_scale, unsigned* status,
                           cudaStream_t stream) {
    PrepGroup grp = {};
    grp.W[0] = W;
    grp.packed[0] = packed;
    grp.row_scale[0] = row_scale;
    grp.mask_bits[0] = mask_bits;
    grp.row_end[0] = O;
    grp.G = 1;
    launch_prep_group<M, N>(grp, K, mask_bits != nullptr, scale_bf16, ext_scale, status, stream);
}

// ---------------------------------------------------------------- global scale
// The guide's module listing takes one scale for the whole matrix, the mean of
// |W| over every weight (masked ones included).  The sum is formed exactly with
// the limb columns above: every warp adds its share into per-lane columns in
// shared memory, sums its lanes and adds the ten column totals to global
// columns (64-bit atomics; a column stays below 2^64 while O * K < 2^32).  A
// single thread then resolves the carries, rounds once to double, divides by
// O * K in double and rounds to float, clamps at 1e-5 and, if asked, rounds to
// bf16.  The ternarisation kernels then read that scale instead of their own.
__global__ void __launch_bounds__(kPrepWarps * 32) abs_sum_kernel(const float* __restrict__ W, long long total,
                                                                  unsigned long long* __restrict__ cols,
                                                                  unsigned* status) {
    __shared__ unsigned long long limbs[kPrepWarps][kLimbs][32];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    unsigned long long* my = &limbs[warp][0][lane];
#pragma unroll
    for (int l = 0; l < kLimbs; ++l) my[l * 32] = 0ull;
    bool bad = false;
    const long long nvec = total >> 2;  // K % 16 == 0, so whole float4 vectors
    const uint4* w4 = reinterpret_cast<const uint4*>(W);
    for (long long v = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; v < nvec;
         v += static_cast<long long>(gridDim.x) * blockDim.x) {
        const uint4 q = ldg_nc(w4 + v);
        const uint32_t a[4] = {q.x & 0x7FFFFFFFu, q.y & 0x7FFFFFFFu, q.z & 0x7FFFFFFFu, q.w & 0x7FFFFFFFu};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            bad |= a[i] >= 0x7F800000u;
            if (a[i] < 0x7F800000u) exact_add(my, a[i]);
        }
    }
    if (bad) raise_status(status, kStatusNonfinite);
    __syncwarp();
    if (lane < kLimbs) {
        unsigned long long s = 0;
        for (int i = 0; i < 32; ++i) s += limbs[warp][lane][i];
        if (s) atomicAdd(cols + lane, s);
    }
}

__global__ void gamma_finalize_kernel(const unsigned long long* __restrict__ cols, long long total, int scale_bf16,
                                      float* __restrict__ gamma) {
    if (threadIdx.x != 0 || blockIdx.x != 0) return;
    uint32_t w[kLimbs];
    unsigned long long carry = 0;
#pragma unroll
    for (int i = 0; i < kLimbs; ++i) {
        const unsigned long long lo = cols[i] & 0xFFFFFFFFull, hi = cols[i] >> 32;
        const unsigned long long t = lo + carry;
        w[i] = static_cast<uint32_t>(t);
        carry = (t >> 32) + hi;
    }
    const double sum = limbs_to_double(w);
    *gamma = scale_storage(fmaxf(__double2float_rn(__ddiv_rn(sum, static_cast<double>(total))), 1e-5f), scale_bf16);
}

// Per-device scratch of the global-scale path: ten columns and the scale.  Calls
// that use it on one device must be ordered (one stream, or synchronised).
__device__ unsigned long long g_gamma_cols[kLimbs];
__device__ float g_gamma;

cudaError_t launch_prep(const float* W, long long O, long long K, int n, int m, uint8_t* packed, float* row_scale,
                        uint8_t* mask_bits, int scale_bf16, int scale_global, unsigned* status, cudaStream_t stream) {
    const float* ext = nullptr;
    if (scale_global) {
        unsigned long long* cols = nullptr;
        float* gamma = nullptr;
        cudaError_t e = cudaGetSymbolAddress(reinterpret_cast<void**>(&cols), g_gamma_cols);
        if (e == cudaSuccess) e = cudaGetSymbolAddress(reinterpret_cast<void**>(&gamma), g_gamma);
        if (e == cudaSuccess) e = cudaMemsetAsync(cols, 0, sizeof(unsigned long long) * kLimbs, stream);
        if (e != cudaSuccess) return e;
        const long long total = O * K;
        long long blocks = (total / 4 + kPrepWarps * 32 - 1) / (kPrepWarps * 32);
        if (blocks > 4096) blocks = 4096;
        abs_sum_kernel<<<static_cast<unsigned>(blocks), kPrepWarps * 32, 0, stream>>>(W, total, cols, status);
        gamma_finalize_kernel<<<1, 32, 0, stream>>>(cols, total, scale_bf16, gamma);
        ext = gamma;
    }
    if (m == 4 && n == 2) launch_prep_mn<4, 2>(W, O, K, packed, row_scale, mask_bits, scale_bf16, ext, status, stream);
    else if (m == 4) launch_prep_mn<4, 3>(W, O, K, packed, row_scale, mask_bits, scale_bf16, ext, status, stream);
    else if (n == 4) launch_prep_mn<8, 4>(W, O, K, packed, row_scale, mask_bits, scale_bf16, ext, status, stream);
    else launch_prep_mn<8, 6>(W, O, K, packed, row_scale, mask_bits, scale_bf16, ext, status, stream);
    return cudaGetLastError();
}

int prep_max_group() { return kPrepMaxGroup; }

// G matrices of equal K, per-row scales (no flags), in one launch when their
// rows fit the register-resident kernel (K <= 8192).  mask_bits may be null,
// or hold null entries.
cudaError_t launch_prep_grouped(int G, const float* const* W, const long long* O, long long K, int n, int m,
                                uint8_t* const* packed, float* const* row_scale, uint8_t* const* mask_bits,
                                unsigned* status, cudaStream_t stream) {
    if (G < 1 || G > kPrepMaxGroup) return cudaErrorInvalidValue;
    PrepGroup grp = {};
    long long end = 0;
    bool with_mask = false;
    for (int g = 0; g < G; ++g) {
        grp.W[g] = W[g];
        grp.packed[g] = packed[g];
        grp.row_scale[g] = row_scale[g];
        grp.mask_bits[g] = mask_bits ? mask_bits[g] : nullptr;
        with_mask |= grp.mask_bits[g] != nullptr;
        end += O[g];
        grp.row_end[g] = end;
    }
    grp.G = G;
    if (end == 0) return cudaSuccess;
    if (m == 4 && n == 2) launch_prep_group<4, 2>(grp, K, with_mask, 0, nullptr, status, stream);
    else if (m == 4) launch_prep_group<4, 3>(grp, K, with_mask, 0, nullptr, status, stream);
    else if (n == 4) launch_prep_group<8, 4>(grp, K, with_mask, 0, nullptr, status, stream);
    else launch_prep_group<8, 6>(grp, K, with_mask, 0, nullptr, status, stream);
    return cudaGetLastError();
}

}  // namespace sbl
