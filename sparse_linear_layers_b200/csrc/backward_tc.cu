// Straight-through backward on the tcgen05 tensor cores (kind::f16, bf16
// operands, fp32 accumulators in tensor memory).
//
// The gradients of the Sparse-BitNet Guide's "Training Stability & The
// Straight-Through Estimator" (the backward passes the mask and the ternary
// rounding unchanged), read with every quantiser the identity:
//
//   dX[t, k] = sum_o (dY[t, o] * scale_o) * W_t[o, k]       (M = T, N = K, reduction over O)
//   dW[o, k] = sum_t (dY[t, o] / s_t) * x_q[t, k]           (M = O, N = K, reduction over T)
//
// Both are dense contractions.  One factor is ternary or int8 (|x_q| <= 127),
// exact in bf16; the other is an fp32 value v (dY * scale_o, or dY / s_t, one
// IEEE rounding each, as on the CUDA cores).  v splits exactly into three bf16
// parts: hi = v with its low 16 bits cleared, mid = (v - hi) likewise, lo =
// v - hi - mid (v - hi has at most 16 significant bits and lo at most 8, so
// every difference is exact and every part a bf16).  Each part times a ternary
// or int8 value is exact in fp32, so
//
//   out = sum_r (hi_r + mid_r + lo_r) * b_r
//
// is a bf16 contraction over 3n terms with fp32 accumulation.
//
// Two steps per gradient:
//   1. a pass over memory writes both operands K-major in bf16 into the
//      workspace: A' [M, 3 * np] (the three parts of each row, plane p at
//      columns p * np .. p * np + n - 1, zero padded to np = n rounded up to 64)
//      and B [N, np] (the ternary weights transposed for dX, the int8
//      activations transposed for dW, zero padded);
//   2. a persistent, warp-specialised GEMM: TMA loads, per 64-deep k-block,
//      the three A' planes of 128 rows and one B tile of BN rows (all
//      128B-swizzled, K-major); one thread issues 12 tcgen05.mma kind::f16
//      (M = 128, N = BN, K = 16) into one of two TMEM accumulators; four
//      epilogue warps read the accumulator (tcgen05.ld), scale the rows when
//      asked (the ternary form of dW) and write fp32 rows through TMA stores.
//
// Every wait is bounded (mbar_wait); a CTA that gives up raises the timeout
// status, lets in-flight loads and MMAs finish (bounded), frees its tensor
// memory and exits.
#include <cuda.h>

#include "sbl_common.cuh"
#include "tc_util.cuh"

namespace sbl {

namespace bw {
constexpr int BM = 128;           // rows per tile (MMA M, TMEM lanes)
constexpr int BK = 64;            // bf16 reduction elements per k-block (128 bytes)
constexpr int A_BYTES = BM * 128;  // one plane of the A tile
constexpr int EPI_WARPS = 4;
constexpr int WARP_TMA = 4;
constexpr int WARP_MMA = 5;
constexpr int THREADS = 6 * 32;
constexpr int Y_BYTES = 32 * 128;  // one warp's fp32 output staging box: 32 rows x 32 columns
}  // namespace bw

template <int BN>
struct BwdCfg {
    static constexpr int B_BYTES = BN * 128;
    static constexpr int STAGES = BN == 256 ? 2 : 3;
    static constexpr int TMEM_COLS = 2 * BN;
};

template <int BN>
struct BwdSmem {
    uint8_t a[BwdCfg<BN>::STAGES][3][bw::A_BYTES];  // 1024-byte aligned tiles
    uint8_t b[BwdCfg<BN>::STAGES][BwdCfg<BN>::B_BYTES];
    uint8_t ystage[bw::EPI_WARPS][2][bw::Y_BYTES];
    uint64_t full[BwdCfg<BN>::STAGES];
    uint64_t empty[BwdCfg<BN>::STAGES];
    uint64_t tmem_full[2];
    uint64_t tmem_empty[2];
    uint64_t mma_done;
    uint32_t tmem_base;
    int abort_flag;
};

template <int BN>
constexpr size_t bwd_smem_bytes() {
    return sizeof(BwdSmem<BN>) + 1024;
}
static_assert(bwd_smem_bytes<256>() <= 232448, "backward tile does not fit in shared memory");
static_assert(bwd_smem_bytes<128>() <= 232448, "backward tile does not fit in shared memory");

// Instruction descriptor: bf16 x bf16 -> f32, both K-major, M x N.
template <int M, int N>
__device__ __forceinline__ uint32_t bf16_idesc() {
    return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(N >> 3) << 17) |
           (static_cast<uint32_t>(M >> 4) << 24);
}

__device__ __forceinline__ void tc_mma_f16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                           uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(acc)
        : "memory");
}

// out[M, N] (fp32, row-major) = sum over r < 3 * np of A'[m, r] * B[n, r mod np],
// each row then multiplied by row_mul[m] when row_mul is not null.
template <int BN>
__global__ void __launch_bounds__(bw::THREADS, 1)
    bwd_gemm_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
                    const __grid_constant__ CUtensorMap tmap_y, int M, int N, int np,
                    const float* __restrict__ row_mul, unsigned* status) {
    using Cfg = BwdCfg<BN>;
    extern __shared__ uint8_t smem_raw[];
    auto* sm = reinterpret_cast<BwdSmem<BN>*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    volatile int* abort_flag = &sm->abort_flag;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    asm volatile("griddepcontrol.launch_dependents;");
    if (threadIdx.x == 32) {
        prefetch_tmap(&tmap_a);
        prefetch_tmap(&tmap_b);
        prefetch_tmap(&tmap_y);
    }
    const int MT = (M + bw::BM - 1) / bw::BM;
    const int NT = (N + BN - 1) / BN;
    const int tiles = MT * NT;
    const int KB = np / bw::BK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < Cfg::STAGES; ++s) {
            mbar_init(&sm->full[s], 1);
            mbar_init(&sm->empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&sm->tmem_full[b], 1);
            mbar_init(&sm->tmem_empty[b], bw::EPI_WARPS * 32);
        }
        mbar_init(&sm->mma_done, 1);
        sm->abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == bw::WARP_MMA) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&sm->tmem_base)),
                     "r"(Cfg::TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = sm->tmem_base;
    // the operands come from the preceding pass over memory
    asm volatile("griddepcontrol.wait;" ::: "memory");

    auto give_up = [&]() {
        if (!*abort_flag) {
            *abort_flag = 1;
            raise_status(status, kStatusTimeout);
        }
    };

    if (warp < bw::EPI_WARPS) {
        // ------------------------------------------------------------ epilogue
        // Warp w owns TMEM lanes 32w .. 32w + 31 (32 rows of the tile).  Each
        // 32-column slice goes through one of the warp's two 128B-swizzled
        // staging boxes and out by one TMA store (clipped at the ragged edges),
        // with the next slice's tcgen05.ld in flight.
        constexpr int NSL = BN / 32;
        const uint32_t lane_addr = static_cast<uint32_t>(warp * 32) << 16;
        uint32_t nstore = 0;
        int tc = 0;
        for (int tile = blockIdx.x; tile < tiles; tile += gridDim.x, ++tc) {
            const int nt = tile % NT, mt = tile / NT;
            const int b = tc & 1;
            const uint32_t aph = (tc >> 1) & 1;
            if (!warp_wait(&sm->tmem_full[b], aph, abort_flag)) { give_up(); break; }
            tc_fence_after();
            const int m = mt * bw::BM + warp * 32 + lane;
            const float mul = (row_mul && m < M) ? __ldg(row_mul + m) : 1.0f;
            const uint32_t tbase = tmem_base + lane_addr + b * BN;
            uint32_t ra[32], rb[32];
            tmem_ld32_nowait(tbase, ra);
            tmem_ld_wait();
            auto slice = [&](const int k, uint32_t (&cur)[32], uint32_t (&nxt)[32]) {
                const bool more = k + 1 < NSL;
                if (more) {
                    tmem_ld32_nowait(tbase + 32 * (k + 1), nxt);
                } else {
                    tc_fence_before();
                    mbar_arrive(&sm->tmem_empty[b]);  // the accumulator buffer is free for the MMA
                }
                if (row_mul) {
#pragma unroll
                    for (int i = 0; i < 32; ++i) cur[i] = __float_as_uint(__fmul_rn(__uint_as_float(cur[i]), mul));
                }
                uint8_t* const box = sm->ystage[warp][nstore & 1];
                if (lane == 0) bulk_wait_read<1>();
                __syncwarp();
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const uint32_t a = smem_u32(box + lane * 128 + ((c ^ (lane & 7)) << 4));
                    asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(a), "r"(cur[4 * c]), "r"(cur[4 * c + 1]),
                                 "r"(cur[4 * c + 2]), "r"(cur[4 * c + 3])
                                 : "memory");
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) tma_store_2d(&tmap_y, smem_u32(box), nt * BN + 32 * k, mt * bw::BM + warp * 32);
                ++nstore;
                if (more) tmem_ld_wait();
            };
            for (int k = 0; k < NSL; k += 2) {
                slice(k, ra, rb);
                slice(k + 1, rb, ra);
            }
        }
        if (lane == 0) bulk_wait_all();
    } else if (warp == bw::WARP_TMA) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            uint32_t it = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < tiles && ok; tile += gridDim.x) {
                const int nt = tile % NT, mt = tile / NT;
                for (int kb = 0; kb < KB; ++kb, ++it) {
                    const int s = it % Cfg::STAGES;
                    const uint32_t ph = (it / Cfg::STAGES) & 1;
                    if (!mbar_wait(&sm->empty[s], ph ^ 1, abort_flag)) { give_up(); ok = false; break; }
                    mbar_arrive_expect_tx(&sm->full[s], 3 * bw::A_BYTES + Cfg::B_BYTES);
#pragma unroll
                    for (int p = 0; p < 3; ++p)
                        tma_load_2d(smem_u32(sm->a[s][p]), &tmap_a, p * np + kb * bw::BK, mt * bw::BM, &sm->full[s]);
                    tma_load_2d(smem_u32(sm->b[s]), &tmap_b, kb * bw::BK, nt * BN, &sm->full[s]);
                }
            }
            // let every issued load land before the CTA can exit
            const uint32_t first = it > Cfg::STAGES ? it - Cfg::STAGES : 0;
            volatile int never = 0;
            for (uint32_t j = first; j < it; ++j)
                if (!mbar_wait(&sm->full[j % Cfg::STAGES], (j / Cfg::STAGES) & 1, &never)) give_up();
        }
    } else {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t idesc = bf16_idesc<bw::BM, BN>();
            uint32_t it = 0;
            int tc = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < tiles && ok; tile += gridDim.x, ++tc) {
                const int b = tc & 1;
                const uint32_t aph = (tc >> 1) & 1;
                if (!mbar_wait(&sm->tmem_empty[b], aph ^ 1, abort_flag)) { give_up(); break; }
                tc_fence_after();
                const uint32_t d = tmem_base + b * BN;
                for (int kb = 0; kb < KB; ++kb, ++it) {
                    const int s = it % Cfg::STAGES;
                    const uint32_t ph = (it / Cfg::STAGES) & 1;
                    if (!mbar_wait(&sm->full[s], ph, abort_flag)) { give_up(); ok = false; break; }
                    tc_fence_after();
                    const uint32_t b0 = smem_u32(sm->b[s]);
#pragma unroll
                    for (int p = 0; p < 3; ++p) {
                        const uint32_t a0 = smem_u32(sm->a[s][p]);
#pragma unroll
                        for (int kk = 0; kk < bw::BK / 16; ++kk)
                            tc_mma_f16(d, sw128_desc(a0 + kk * 32), sw128_desc(b0 + kk * 32), idesc,
                                       (kb | p | kk) != 0);
                    }
                    tc_commit(&sm->empty[s]);
                }
                if (ok) tc_commit(&sm->tmem_full[b]);
            }
            tc_commit(&sm->mma_done);
            volatile int never = 0;
            if (!mbar_wait(&sm->mma_done, 0, &never)) give_up();
        }
        __syncwarp();
    }

    tc_fence_before();
    __syncthreads();
    if (warp == bw::WARP_MMA) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(Cfg::TMEM_COLS)
                     : "memory");
    }
}

// ---------------------------------------------------------------- operand passes
// The three bf16 parts of v (v = hi + mid + lo exactly; see the file header).
__device__ __forceinline__ void split3(float v, uint16_t& hi, uint16_t& mid, uint16_t& lo) {
    const uint32_t hb = __float_as_uint(v) & 0xFFFF0000u;
    const float r = __fsub_rn(v, __uint_as_float(hb));
    const uint32_t mb = __float_as_uint(r) & 0xFFFF0000u;
    const float l = __fsub_rn(r, __uint_as_float(mb));
    hi = static_cast<uint16_t>(hb >> 16);
    mid = static_cast<uint16_t>(mb >> 16);
    lo = static_cast<uint16_t>(__float_as_uint(l) >> 16);
}

// dX operand A': row t holds the parts of dY[t, o] * scale_o at columns
// p * np + o, zero for O <= o < np.  One thread per pair of columns; the
// grid's rows stride over the tokens.
__global__ void __launch_bounds__(256) bwd_split_dx_kernel(const float* __restrict__ dY,
                                                           const float* __restrict__ row_scale, int T, int O,
                                                           int np, uint16_t* __restrict__ a) {
    asm volatile("griddepcontrol.launch_dependents;");
    asm volatile("griddepcontrol.wait;" ::: "memory");
    for (int t = blockIdx.y; t < T; t += gridDim.y) {
    const size_t row = static_cast<size_t>(t) * 3 * np;
    for (int o = 2 * (blockIdx.x * blockDim.x + threadIdx.x); o < np; o += 2 * gridDim.x * blockDim.x) {
        uint16_t h[2] = {0, 0}, m[2] = {0, 0}, l[2] = {0, 0};
#pragma unroll
        for (int j = 0; j < 2; ++j)
            if (o + j < O)
                split3(__fmul_rn(__ldg(dY + static_cast<size_t>(t) * O + o + j), __ldg(row_scale + o + j)), h[j], m[j],
                       l[j]);
        *reinterpret_cast<uint32_t*>(a + row + o) = h[0] | (static_cast<uint32_t>(h[1]) << 16);
        *reinterpret_cast<uint32_t*>(a + row + np + o) = m[0] | (static_cast<uint32_t>(m[1]) << 16);
        *reinterpret_cast<uint32_t*>(a + row + 2 * np + o) = l[0] | (static_cast<uint32_t>(l[1]) << 16);
    }
    }
}

// dW operand A': row o holds the parts of dY[t, o] / s_t at columns p * np + t,
// zero for T <= t < np.  32 x 32 tiles transposed through shared memory.
__global__ void __launch_bounds__(256) bwd_split_dw_kernel(const float* __restrict__ dY,
                                                           const float* __restrict__ s_tok, int T, int O, int np,
                                                           uint16_t* __restrict__ a) {
    __shared__ uint16_t part[3][32][34];
    asm volatile("griddepcontrol.launch_dependents;");
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
    const int o0 = blockIdx.x * 32, t0 = blockIdx.y * 32;
#pragma unroll
    for (int j = ty; j < 32; j += 8) {
        const int t = t0 + j, o = o0 + tx;
        uint16_t h = 0, m = 0, l = 0;
        if (t < T && o < O) split3(__fdiv_rn(__ldg(dY + static_cast<size_t>(t) * O + o), __ldg(s_tok + t)), h, m, l);
        part[0][tx][j] = h;
        part[1][tx][j] = m;
        part[2][tx][j] = l;
    }
    __syncthreads();
#pragma unroll
    for (int j = ty; j < 32; j += 8) {
        const int o = o0 + j, t = t0 + tx;
        if (o < O && t < np) {
            const size_t row = static_cast<size_t>(o) * 3 * np;
            a[row + t] = part[0][j][tx];
            a[row + np + t] = part[1][j][tx];
            a[row + 2 * np + t] = part[2][j][tx];
        }
    }
}

// dX operand B: row k holds W_t[o, k] (0, +1, -1 as bf16) at column o, zero
// for O <= o < np.  32 x 32 tiles transposed through shared memory.
__global__ void __launch_bounds__(256) bwd_codes_t_kernel(const uint8_t* __restrict__ packed, int O, int K, int np,
                                                          uint16_t* __restrict__ bt) {
    __shared__ uint16_t tile[32][34];
    asm volatile("griddepcontrol.launch_dependents;");
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
    const int k0 = blockIdx.x * 32, o0 = blockIdx.y * 32;
#pragma unroll
    for (int j = ty; j < 32; j += 8) {
        const int o = o0 + j, k = k0 + tx;
        uint16_t v = 0;
        if (o < O && k < K) {
            const uint32_t c = (__ldg(packed + static_cast<size_t>(o) * (K / 4) + k / 4) >> (2 * (k & 3))) & 3u;
            v = c == 1u ? 0x3F80u : (c == 2u ? 0xBF80u : 0u);
        }
        tile[tx][j] = v;
    }
    __syncthreads();
#pragma unroll
    for (int j = ty; j < 32; j += 8) {
        const int k = k0 + j, o = o0 + tx;
        if (k < K && o < np) bt[static_cast<size_t>(k) * np + o] = tile[j][tx];
    }
}

// dW operand B: row k holds x_q[t, k] as bf16 at column t, zero for T <= t < np.
__global__ void __launch_bounds__(256) bwd_xq_t_kernel(const int8_t* __restrict__ xq, int T, int K, int np,
                                                       uint16_t* __restrict__ bt) {
    __shared__ uint16_t tile[32][34];
    asm volatile("griddepcontrol.launch_dependents;");
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
    const int k0 = blockIdx.x * 32, t0 = blockIdx.y * 32;
#pragma unroll
    for (int j = ty; j < 32; j += 8) {
        const int t = t0 + j, k = k0 + tx;
        uint16_t v = 0;
        if (t < T && k < K) v = __bfloat16_as_ushort(__float2bfloat16_rn(static_cast<float>(xq[static_cast<size_t>(t) * K + k])));
        tile[tx][j] = v;
    }
    __syncthreads();
#pragma unroll
    for (int j = ty; j < 32; j += 8) {
        const int k = k0 + j, t = t0 + tx;
        if (k < K && t < np) bt[static_cast<size_t>(k) * np + t] = tile[j][tx];
    }
}

// ---------------------------------------------------------------- host side
static long long pad64(long long n) { return (n + 63) / 64 * 64; }
static size_t round256(size_t b) { return (b + 255) / 256 * 256; }

// Workspace of one gradient: A' [M, 3 * np] and B [N, np], bf16.
static size_t grad_ws_bytes(long long M, long long N, long long n) {
    const long long np = pad64(n > 0 ? n : 1);
    return round256(static_cast<size_t>(M) * 3 * np * 2) + round256(static_cast<size_t>(N) * np * 2);
}

size_t backward_tc_workspace_bytes(long long T, long long O, long long K, int need_dx, int need_dw) {
    size_t b = 0;
    if (need_dx && T > 0 && O > 0) b = grad_ws_bytes(T, K, O);
    if (need_dw && T > 0 && O > 0) {
        const size_t w = grad_ws_bytes(O, K, T);
        b = w > b ? w : b;
    }
    return b;
}

template <typename F, typename... Args>
static cudaError_t launch_pdl(F kernel, dim3 grid, dim3 block, size_t smem, cudaStream_t stream, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, args...);
}

template <int BN>
static cudaError_t launch_bwd_gemm(const uint16_t* a, const uint16_t* b, float* out, long long M, long long N,
                                   long long np, const float* row_mul, unsigned* status, int num_sms,
                                   cudaStream_t stream) {
    EncodeTiledFn enc = get_encode_fn();
    if (!enc) return cudaErrorNotSupported;
    const cuuint32_t estr[2] = {1, 1};
    CUtensorMap map_a, map_b, map_y;
    {
        const cuuint64_t dims[2] = {static_cast<cuuint64_t>(3 * np), static_cast<cuuint64_t>(M)};
        const cuuint64_t strides[1] = {static_cast<cuuint64_t>(3 * np * 2)};
        const cuuint32_t box[2] = {static_cast<cuuint32_t>(bw::BK), static_cast<cuuint32_t>(bw::BM)};
        if (enc(&map_a, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(a), dims, strides, box, estr,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    {
        const cuuint64_t dims[2] = {static_cast<cuuint64_t>(np), static_cast<cuuint64_t>(N)};
        const cuuint64_t strides[1] = {static_cast<cuuint64_t>(np * 2)};
        const cuuint32_t box[2] = {static_cast<cuuint32_t>(bw::BK), static_cast<cuuint32_t>(BN)};
        if (enc(&map_b, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(b), dims, strides, box, estr,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    {
        const cuuint64_t dims[2] = {static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(M)};
        const cuuint64_t strides[1] = {static_cast<cuuint64_t>(N * 4)};
        const cuuint32_t box[2] = {32u, 32u};
        if (enc(&map_y, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, out, dims, strides, box, estr,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    constexpr size_t smem = bwd_smem_bytes<BN>();
    static bool attr_set[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64 || !attr_set[dev]) {
        cudaError_t e = cudaFuncSetAttribute(bwd_gemm_kernel<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(smem));
        if (e != cudaSuccess) return e;
        if (dev >= 0 && dev < 64) attr_set[dev] = true;
    }
    const long long tiles = ((M + bw::BM - 1) / bw::BM) * ((N + BN - 1) / BN);
    const int grid = static_cast<int>(tiles < num_sms ? tiles : num_sms);
    return launch_pdl(bwd_gemm_kernel<BN>, dim3(grid), dim3(bw::THREADS), smem, stream, map_a, map_b, map_y,
                      static_cast<int>(M), static_cast<int>(N), static_cast<int>(np), row_mul, status);
}

static cudaError_t launch_gemm(const uint16_t* a, const uint16_t* b, float* out, long long M, long long N,
                               long long np, const float* row_mul, unsigned* status, int num_sms, cudaStream_t stream) {
    // 256-wide tiles unless they leave more than a quarter of the SMs idle
    const long long mt = (M + bw::BM - 1) / bw::BM;
    const long long wide = mt * ((N + 255) / 256), narrow = mt * ((N + 127) / 128);
    if (N > 128 && (wide >= num_sms || 4 * wide >= 3 * (narrow < num_sms ? narrow : num_sms)))
        return launch_bwd_gemm<256>(a, b, out, M, N, np, row_mul, status, num_sms, stream);
    return launch_bwd_gemm<128>(a, b, out, M, N, np, row_mul, status, num_sms, stream);
}

// dX and/or dW on the tensor cores.  Sizes are validated by the caller
// (T, O > 0; K % 16 == 0; int32-range extents); ws holds
// backward_tc_workspace_bytes() bytes, 256-byte aligned.
cudaError_t launch_backward_tc(const float* dY, long long T, long long O, const int8_t* xq, const float* s_tok,
                               long long K, const uint8_t* packed, const float* row_scale, float* dX, float* dW,
                               int dw_ternary, void* ws, unsigned* status, int num_sms, cudaStream_t stream) {
    uint8_t* base = static_cast<uint8_t*>(ws);
    cudaError_t e = cudaSuccess;
    if (dX) {
        const long long np = pad64(O);
        uint16_t* a = reinterpret_cast<uint16_t*>(base);
        uint16_t* b = reinterpret_cast<uint16_t*>(base + round256(static_cast<size_t>(T) * 3 * np * 2));
        const int per_row = static_cast<int>((np / 2 + 255) / 256);
        e = launch_pdl(bwd_split_dx_kernel, dim3(per_row, static_cast<unsigned>(T < 65535 ? T : 65535)), dim3(256), 0,
                       stream, dY,
                       row_scale, static_cast<int>(T), static_cast<int>(O), static_cast<int>(np), a);
        if (e != cudaSuccess) return e;
        e = launch_pdl(bwd_codes_t_kernel, dim3(static_cast<unsigned>((K + 31) / 32), static_cast<unsigned>((np + 31) / 32)),
                       dim3(256), 0, stream, packed, static_cast<int>(O), static_cast<int>(K), static_cast<int>(np), b);
        if (e != cudaSuccess) return e;
        e = launch_gemm(a, b, dX, T, K, np, nullptr, status, num_sms, stream);
        if (e != cudaSuccess) return e;
    }
    if (dW) {
        const long long np = pad64(T);
        uint16_t* a = reinterpret_cast<uint16_t*>(base);
        uint16_t* b = reinterpret_cast<uint16_t*>(base + round256(static_cast<size_t>(O) * 3 * np * 2));
        e = launch_pdl(bwd_split_dw_kernel, dim3(static_cast<unsigned>((O + 31) / 32), static_cast<unsigned>((np + 31) / 32)),
                       dim3(256), 0, stream, dY, s_tok, static_cast<int>(T), static_cast<int>(O), static_cast<int>(np), a);
        if (e != cudaSuccess) return e;
        e = launch_pdl(bwd_xq_t_kernel, dim3(static_cast<unsigned>((K + 31) / 32), static_cast<unsigned>((np + 31) / 32)),
                       dim3(256), 0, stream, xq, static_cast<int>(T), static_cast<int>(K), static_cast<int>(np), b);
        if (e != cudaSuccess) return e;
        e = launch_gemm(a, b, dW, O, K, np, dw_ternary ? row_scale : nullptr, status, num_sms, stream);
    }
    return e;
}

}  // namespace sbl
