// Prefill path: acc[t, o] = sum_k x_q[t, k] * W_t[o, k] on the tcgen05 tensor
// cores (kind::i8, int32 accumulators in tensor memory), then y = acc * scale_o / s_t.
//
// The contraction of the Sparse-BitNet Guide's linear-evaluation equation
// ("Mathematical Formulation of Sparse-BitLinear"), which for many tokens is a
// dense int8 matrix product.  Persistent, warp-specialised, one CTA per SM:
//
//   warps 0-3          epilogue: tcgen05.ld of the accumulator (TMEM lane = token),
//                      dequantise, 16-byte stores of y rows (contiguous in o)
//   warps 4..4+BN/32-1 weight expansion: each thread owns one output row o of
//                      the B tile, loads its 2-bit codes for the k-block and
//                      writes the int8 row into the 128B-swizzled K-major tile
//   next warp          TMA producer of the activation tile (A, 128 tokens x 128 k)
//   last warp          TMEM allocator and single-thread MMA issuer
//
// Tile: 128 tokens x BN output rows x 128 k per stage, 4 stages, two TMEM
// accumulator buffers so the epilogue of one tile overlaps the MMAs of the next.
// The weights are expanded in the interleaved 16-element order of
// expand_codes(); the activations were quantised into the same order.
//
// Every wait is bounded (mbar_wait); a CTA that gives up raises the timeout
// status, lets in-flight TMA loads and MMAs finish (bounded), frees its tensor
// memory and exits.
#include <cuda.h>

#include "sbl_common.cuh"

namespace sbl {

namespace pf {
constexpr int BM = 128;       // tokens per tile  (MMA M, TMEM lanes)
constexpr int BK = 128;       // k per stage      (bytes of int8)
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BK;
constexpr int EPI_WARPS = 4;
}  // namespace pf

template <int BN>
struct PrefillCfg {
    static constexpr int B_BYTES = BN * pf::BK;
    static constexpr int DEC_WARPS = BN / 32;
    static constexpr int WARP_TMA = pf::EPI_WARPS + DEC_WARPS;
    static constexpr int WARP_MMA = WARP_TMA + 1;
    static constexpr int THREADS = (WARP_MMA + 1) * 32;
    static constexpr int TMEM_COLS = 2 * BN;  // two accumulator buffers
};

template <int BN>
struct PrefillSmem {
    uint8_t a[pf::STAGES][pf::A_BYTES];            // 1024-byte aligned tiles
    uint8_t b[pf::STAGES][PrefillCfg<BN>::B_BYTES];
    uint64_t full_tma[pf::STAGES];
    uint64_t full_dec[pf::STAGES];
    uint64_t empty[pf::STAGES];
    uint64_t tmem_full[2];
    uint64_t tmem_empty[2];
    uint64_t mma_done;
    uint32_t tmem_base;
    int abort_flag;
};

template <int BN>
constexpr size_t prefill_smem_bytes() {
    return sizeof(PrefillSmem<BN>) + 1024;
}

// UMMA shared-memory descriptor: K-major, 128-byte swizzle, 8-row groups 1024 B apart.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
    uint64_t d = static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
    d |= static_cast<uint64_t>(1u) << 16;            // leading byte offset (unused for this layout)
    d |= static_cast<uint64_t>(1024u >> 4) << 32;    // stride byte offset
    d |= static_cast<uint64_t>(1u) << 46;            // descriptor version
    d |= static_cast<uint64_t>(2u) << 61;            // SWIZZLE_128B
    return d;
}

// Instruction descriptor: s8 x s8 -> s32, both K-major, M = 128, N = BN.
template <int BN>
__device__ __forceinline__ uint32_t i8_idesc() {
    return (2u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(BN >> 3) << 17) |
           (static_cast<uint32_t>(pf::BM >> 4) << 24);
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
            dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(acc)
        : "memory");
}

__device__ __forceinline__ void tc_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void st_v4(void* p, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    asm volatile("st.global.v4.b32 [%0], {%1,%2,%3,%4};" ::"l"(p), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

template <int BN>
__global__ void __launch_bounds__(PrefillCfg<BN>::THREADS, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap tmap_x, const uint8_t* __restrict__ packed,
                   const float* __restrict__ row_scale, const float* __restrict__ s_tok, int T, int O, int K,
                   void* __restrict__ y, int y_bf16, int32_t* __restrict__ acc_out, unsigned* status) {
    using Cfg = PrefillCfg<BN>;
    extern __shared__ uint8_t smem_raw[];
    auto* sm = reinterpret_cast<PrefillSmem<BN>*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    volatile int* abort_flag = &sm->abort_flag;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int MT = (T + pf::BM - 1) / pf::BM;
    const int NT = (O + BN - 1) / BN;
    const int tiles = MT * NT;
    const int KB = (K + pf::BK - 1) / pf::BK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < pf::STAGES; ++s) {
            mbar_init(&sm->full_tma[s], 1);
            mbar_init(&sm->full_dec[s], Cfg::DEC_WARPS * 32);
            mbar_init(&sm->empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&sm->tmem_full[b], 1);
            mbar_init(&sm->tmem_empty[b], pf::EPI_WARPS * 32);
        }
        mbar_init(&sm->mma_done, 1);
        sm->abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == Cfg::WARP_MMA) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&sm->tmem_base)),
                     "r"(Cfg::TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = sm->tmem_base;

    auto give_up = [&]() {
        if (!*abort_flag) {
            *abort_flag = 1;
            raise_status(status, kStatusTimeout);
        }
    };

    if (warp < pf::EPI_WARPS) {
        // ------------------------------------------------------------ epilogue
        const int row = threadIdx.x;  // TMEM lane == token within the tile
        int tc = 0;
        for (int tile = blockIdx.x; tile < tiles; tile += gridDim.x, ++tc) {
            const int mt = tile % MT, nt = tile / MT;
            const int b = tc & 1;
            const uint32_t aph = (tc >> 1) & 1;
            // warp-uniform decision: tcgen05.ld below is a .sync.aligned warp instruction
            const bool ready = __all_sync(0xFFFFFFFFu, mbar_wait(&sm->tmem_full[b], aph, abort_flag));
            if (!ready) { give_up(); break; }
            tc_fence_after();
            const int t = mt * pf::BM + row;
            const bool tvalid = t < T;
            const float inv_s = tvalid ? __frcp_rn(s_tok[t]) : 0.f;
            for (int q = 0; q < BN / 32; ++q) {
                uint32_t r[32];
                tmem_ld32(tmem_base + (static_cast<uint32_t>(warp * 32) << 16) + b * BN + q * 32, r);
                if (q == BN / 32 - 1) {
                    tc_fence_before();
                    mbar_arrive(&sm->tmem_empty[b]);
                }
                const int o0 = nt * BN + q * 32;
                if (!tvalid || o0 >= O) continue;
                const long long base = static_cast<long long>(t) * O + o0;
                const bool full = (o0 + 32 <= O) && ((O & 3) == 0);
                float v[32];
#pragma unroll
                for (int i = 0; i < 32; i += 4) {
                    float4 sc = make_float4(0.f, 0.f, 0.f, 0.f);
                    if (full) sc = __ldg(reinterpret_cast<const float4*>(row_scale + o0 + i));
                    else {
                        if (o0 + i + 0 < O) sc.x = row_scale[o0 + i + 0];
                        if (o0 + i + 1 < O) sc.y = row_scale[o0 + i + 1];
                        if (o0 + i + 2 < O) sc.z = row_scale[o0 + i + 2];
                        if (o0 + i + 3 < O) sc.w = row_scale[o0 + i + 3];
                    }
                    v[i + 0] = __fmul_rn(__fmul_rn(static_cast<float>(static_cast<int>(r[i + 0])), sc.x), inv_s);
                    v[i + 1] = __fmul_rn(__fmul_rn(static_cast<float>(static_cast<int>(r[i + 1])), sc.y), inv_s);
                    v[i + 2] = __fmul_rn(__fmul_rn(static_cast<float>(static_cast<int>(r[i + 2])), sc.z), inv_s);
                    v[i + 3] = __fmul_rn(__fmul_rn(static_cast<float>(static_cast<int>(r[i + 3])), sc.w), inv_s);
                }
                if (full) {
                    if (y_bf16) {
                        uint32_t p[16];
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            const __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
                            p[i] = *reinterpret_cast<const uint32_t*>(&h);
                        }
                        uint16_t* yp = reinterpret_cast<uint16_t*>(y) + base;
#pragma unroll
                        for (int i = 0; i < 16; i += 4) st_v4(yp + 2 * i, p[i], p[i + 1], p[i + 2], p[i + 3]);
                    } else {
                        float* yp = reinterpret_cast<float*>(y) + base;
#pragma unroll
                        for (int i = 0; i < 32; i += 4)
                            st_v4(yp + i, __float_as_uint(v[i]), __float_as_uint(v[i + 1]), __float_as_uint(v[i + 2]),
                                  __float_as_uint(v[i + 3]));
                    }
                    if (acc_out) {
#pragma unroll
                        for (int i = 0; i < 32; i += 4) st_v4(acc_out + base + i, r[i], r[i + 1], r[i + 2], r[i + 3]);
                    }
                } else {
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        if (o0 + i >= O) continue;
                        if (y_bf16)
                            reinterpret_cast<__nv_bfloat16_raw*>(y)[base + i] =
                                static_cast<__nv_bfloat16_raw>(__float2bfloat16_rn(v[i]));
                        else
                            reinterpret_cast<float*>(y)[base + i] = v[i];
                        if (acc_out) acc_out[base + i] = static_cast<int>(r[i]);
                    }
                }
            }
        }
    } else if (warp < Cfg::WARP_TMA) {
        // ------------------------------------------------------------ weight expansion
        const int r = threadIdx.x - pf::EPI_WARPS * 32;  // row of the B tile
        const int rowbytes = K >> 2;
        uint32_t it = 0;
        bool ok = true;
        for (int tile = blockIdx.x; tile < tiles && ok; tile += gridDim.x) {
            const int nt = tile / MT;
            const int o = nt * BN + r;
            const bool valid = o < O;
            const uint8_t* prow = packed + static_cast<long long>(o) * rowbytes;
            uint4 p0 = make_uint4(0u, 0u, 0u, 0u), p1 = p0;
            if (valid) {
                p0 = ldg_nc(prow);
                if (64 < K) p1 = ldg_nc(prow + 16);
            }
            for (int kb = 0; kb < KB; ++kb, ++it) {
                // prefetch the next k-block's codes before waiting for the slot
                uint4 n0 = make_uint4(0u, 0u, 0u, 0u), n1 = n0;
                const int kn = (kb + 1) * pf::BK;
                if (valid && kn < K) {
                    n0 = ldg_nc(prow + (kn >> 2));
                    if (kn + 64 < K) n1 = ldg_nc(prow + (kn >> 2) + 16);
                }
                const int s = it % pf::STAGES;
                const uint32_t ph = (it / pf::STAGES) & 1;
                if (!mbar_wait(&sm->empty[s], ph ^ 1, abort_flag)) { give_up(); ok = false; break; }
                uint8_t* dst = sm->b[s] + r * 128;
                const int sw = r & 7;
                const uint32_t words[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    uint32_t e[4];
                    expand_codes(words[c], e);
                    const uint32_t a = smem_u32(dst + ((c ^ sw) << 4));
                    asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(a), "r"(e[0]), "r"(e[1]), "r"(e[2]),
                                 "r"(e[3])
                                 : "memory");
                }
                fence_proxy_async_smem();
                mbar_arrive(&sm->full_dec[s]);
                p0 = n0;
                p1 = n1;
            }
        }
    } else if (warp == Cfg::WARP_TMA) {
        // ------------------------------------------------------------ activation TMA producer
        if (lane == 0) {
            uint32_t it = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < tiles && ok; tile += gridDim.x) {
                const int mt = tile % MT;
                for (int kb = 0; kb < KB; ++kb, ++it) {
                    const int s = it % pf::STAGES;
                    const uint32_t ph = (it / pf::STAGES) & 1;
                    if (!mbar_wait(&sm->empty[s], ph ^ 1, abort_flag)) { give_up(); ok = false; break; }
                    mbar_arrive_expect_tx(&sm->full_tma[s], pf::A_BYTES);
                    tma_load_2d(smem_u32(sm->a[s]), &tmap_x, kb * pf::BK, mt * pf::BM, &sm->full_tma[s]);
                }
            }
            // let every issued load land before the CTA can exit
            const uint32_t first = it > pf::STAGES ? it - pf::STAGES : 0;
            volatile int never = 0;
            for (uint32_t j = first; j < it; ++j)
                if (!mbar_wait(&sm->full_tma[j % pf::STAGES], (j / pf::STAGES) & 1, &never)) give_up();
        }
    } else {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t idesc = i8_idesc<BN>();
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
                    const int s = it % pf::STAGES;
                    const uint32_t ph = (it / pf::STAGES) & 1;
                    if (!mbar_wait(&sm->full_tma[s], ph, abort_flag) || !mbar_wait(&sm->full_dec[s], ph, abort_flag)) {
                        give_up();
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a0 = smem_u32(sm->a[s]), b0 = smem_u32(sm->b[s]);
#pragma unroll
                    for (int kk = 0; kk < pf::BK / 32; ++kk)
                        tc_mma(d, sw128_desc(a0 + kk * 32), sw128_desc(b0 + kk * 32), idesc, (kb | kk) != 0);
                    tc_commit(&sm->empty[s]);
                }
                if (ok) tc_commit(&sm->tmem_full[b]);
            }
            // all MMAs must be complete before tensor memory is released
            tc_commit(&sm->mma_done);
            volatile int never = 0;
            if (!mbar_wait(&sm->mma_done, 0, &never)) give_up();
        }
        __syncwarp();
    }

    tc_fence_before();
    __syncthreads();
    if (warp == Cfg::WARP_MMA) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(Cfg::TMEM_COLS)
                     : "memory");
    }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn get_encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

template <int BN>
static cudaError_t launch_prefill_bn(const int8_t* xperm, const float* s_tok, long long T, long long K,
                                     const uint8_t* packed, const float* row_scale, long long O, void* y, int y_bf16,
                                     int32_t* acc_out, unsigned* status, int num_sms, cudaStream_t stream) {
    EncodeTiledFn enc = get_encode_fn();
    if (!enc) return cudaErrorNotSupported;
    CUtensorMap map;
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(T)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(K)};
    const cuuint32_t box[2] = {static_cast<cuuint32_t>(pf::BK), static_cast<cuuint32_t>(pf::BM)};
    const cuuint32_t estr[2] = {1, 1};
    if (enc(&map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<int8_t*>(xperm), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    constexpr size_t smem = prefill_smem_bytes<BN>();
    static bool attr_set[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64 || !attr_set[dev]) {
        cudaError_t e = cudaFuncSetAttribute(prefill_kernel<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(smem));
        if (e != cudaSuccess) return e;
        if (dev >= 0 && dev < 64) attr_set[dev] = true;
    }
    const long long tiles = ((T + pf::BM - 1) / pf::BM) * ((O + BN - 1) / BN);
    const int grid = static_cast<int>(tiles < num_sms ? tiles : num_sms);
    prefill_kernel<BN><<<grid, PrefillCfg<BN>::THREADS, smem, stream>>>(
        map, packed, row_scale, s_tok, static_cast<int>(T), static_cast<int>(O), static_cast<int>(K), y, y_bf16,
        acc_out, status);
    return cudaGetLastError();
}

cudaError_t launch_prefill(const int8_t* xperm, const float* s_tok, long long T, long long K, const uint8_t* packed,
                           const float* row_scale, long long O, void* y, int y_bf16, int32_t* acc_out,
                           unsigned* status, int num_sms, cudaStream_t stream) {
    // Wide tiles halve the expansion work per MMA; narrow ones fill the SMs
    // when there are few tiles.
    const long long mt = (T + pf::BM - 1) / pf::BM;
    const long long wide_tiles = mt * ((O + 255) / 256);
    const long long wide_waves = (wide_tiles + num_sms - 1) / num_sms;
    const long long narrow_tiles = mt * ((O + 127) / 128);
    const long long narrow_waves = (narrow_tiles + num_sms - 1) / num_sms;
    if (2 * wide_waves <= narrow_waves || narrow_waves >= 8)
        return launch_prefill_bn<256>(xperm, s_tok, T, K, packed, row_scale, O, y, y_bf16, acc_out, status, num_sms,
                                      stream);
    return launch_prefill_bn<128>(xperm, s_tok, T, K, packed, row_scale, O, y, y_bf16, acc_out, status, num_sms,
                                  stream);
}

}  // namespace sbl
