// Prefill path: acc[t, o] = sum_k x_q[t, k] * W_t[o, k] on the tcgen05 tensor
// cores (kind::i8, int32 accumulators in tensor memory), then y = acc * scale_o / s_t.
//
// The contraction of the Sparse-BitNet Guide's linear-evaluation equation
// ("Mathematical Formulation of Sparse-BitLinear"), which for many tokens is a
// dense int8 matrix product.  Persistent, warp-specialised, one CTA per SM:
//
//   warps 0-3          epilogue: warp w owns TMEM lanes 32w .. 32w + 31 (32 tokens);
//                      pipelined tcgen05.ld, dequantise, per-warp 128B-swizzled
//                      double-buffered staging boxes, TMA bulk stores
//   warps 4..4+BN/32-1 weight expansion: each thread owns one output row o of
//                      the B tile, reads its 2-bit codes for the k-block from
//                      shared memory and writes the int8 row into the
//                      128B-swizzled K-major tile
//   next warp          TMA producer: activation tile (A, 128 tokens x 128 k) and
//                      the 2-bit code tile (BN rows x 32 bytes) of each stage
//   last warp          TMEM allocator and single-thread MMA issuer
//
// The kernel is launched as a programmatic dependent of the activation
// quantisation: set-up (barriers, tensor memory) overlaps its tail, and every
// role waits on griddepcontrol before touching its outputs.
//
// Tile: 128 tokens x BN output rows x 128 k per stage (3 stages for BN = 256,
// 4 for BN = 128), two TMEM accumulator buffers so the epilogue of one tile
// overlaps the MMAs of the next.  Shared-memory bandwidth is the binding
// resource: per k-block the MMA reads the activation and weight tiles, TMA
// writes the activation and code tiles and the expansion writes the int8
// weight tile (about 112 KB per 128 x 256 x 128 step at BN = 256).
// The weights are expanded in the 16-element pairing order of
// expand_pairs(); the activations were quantised into the same order.
//
// Every wait is bounded (mbar_wait); a CTA that gives up raises the timeout
// status, lets in-flight TMA loads and MMAs finish (bounded), frees its tensor
// memory and exits.
#include <cuda.h>

#include <cstring>
#include <type_traits>

#include "sbl_common.cuh"
#include "tc_util.cuh"

namespace sbl {

#ifdef SBL_TRACE
// Debug builds only: clock64 stamps of pipeline events in CTA 0 (event e,
// iteration i -> g_trace[e * 256 + i]).
__device__ unsigned long long* g_trace;
#define SBL_TR(e, i)                                                          \
    do {                                                                      \
        if (trace_buf && (i) < 256) trace_buf[(e) * 256 + (i)] = clock64();   \
    } while (0)
// per-CTA stamps of event e: global timer at g_trace[e * 256 + b] and clock64
// at g_trace[(e + 20) * 256 + b] for CTA b (the buffer holds 40 x 256 words)
#define SBL_TRB(e)                                                                          \
    do {                                                                                    \
        if (g_trace && blockIdx.x < 256) g_trace[(e) * 256 + blockIdx.x] = global_ns();     \
        if (g_trace && blockIdx.x < 256) g_trace[((e) + 20) * 256 + blockIdx.x] = clock64(); \
    } while (0)
#else
#define SBL_TR(e, i) \
    do {             \
    } while (0)
#define SBL_TRB(e) \
    do {           \
    } while (0)
#endif

namespace pf {
constexpr int BM = 128;       // tokens per tile  (MMA M, TMEM lanes)
constexpr int BK = 128;       // k per stage      (bytes of int8)
constexpr int A_BYTES = BM * BK;
constexpr int EPI_WARPS = 4;
constexpr int Y_BYTES = 32 * 128;  // one warp's output staging box: 32 tokens x 128 bytes
}  // namespace pf

template <int BN>
struct PrefillCfg {
    static constexpr int B_BYTES = BN * pf::BK;
    static constexpr int P_BYTES = BN * pf::BK / 4;  // 2-bit codes of the B tile
    static constexpr int DEC_WARPS = BN / 32;
    static constexpr int WARP_TMA = pf::EPI_WARPS + DEC_WARPS;
    static constexpr int WARP_MMA = WARP_TMA + 1;
    static constexpr int THREADS = (WARP_MMA + 1) * 32;
    static constexpr int TMEM_COLS = 2 * BN;  // two accumulator buffers
    static constexpr int STAGES = BN == 256 ? 3 : 4;
};

template <int BN>
struct PrefillSmem {
    uint8_t a[PrefillCfg<BN>::STAGES][pf::A_BYTES];            // 1024-byte aligned tiles
    uint8_t b[PrefillCfg<BN>::STAGES][PrefillCfg<BN>::B_BYTES];
    uint8_t p[PrefillCfg<BN>::STAGES][PrefillCfg<BN>::P_BYTES];
    uint8_t ystage[pf::EPI_WARPS][2][pf::Y_BYTES];           // per-warp output transpose box
    float wscale[pf::EPI_WARPS][BN];                          // per-warp copy of the tile's row scales
    uint64_t full_tma[PrefillCfg<BN>::STAGES];
    uint64_t full_dec[PrefillCfg<BN>::STAGES];
    uint64_t empty[PrefillCfg<BN>::STAGES];
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
static_assert(prefill_smem_bytes<256>() <= 232448, "prefill tile does not fit in shared memory");
static_assert(prefill_smem_bytes<128>() <= 232448, "prefill tile does not fit in shared memory");

template <int BN, bool GROUPED>
__global__ void __launch_bounds__(PrefillCfg<BN>::THREADS, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ PrefillOut out,
                   const float* __restrict__ s_tok, int T, int K, int y_bf16, int ksplit,
                   int32_t* __restrict__ part, unsigned* status) {
    using Cfg = PrefillCfg<BN>;
    extern __shared__ uint8_t smem_raw[];
    auto* sm = reinterpret_cast<PrefillSmem<BN>*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    volatile int* abort_flag = &sm->abort_flag;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
#ifdef SBL_TRACE
    unsigned long long* const trace_buf = blockIdx.x == 0 ? g_trace : nullptr;
#endif
    asm volatile("griddepcontrol.launch_dependents;");
    if (threadIdx.x == 0) SBL_TR(14, 0);  // kernel entry
    if (threadIdx.x == 0) SBL_TRB(12);
    if (threadIdx.x == 32) {
        prefetch_tmap(&tmap_x);
#pragma unroll
        for (int i = 0; i < (GROUPED ? kPrefillMaxGroup : 1); ++i)
            if (i < out.G) {
                prefetch_tmap(&out.tmap_w[i]);
                prefetch_tmap(&out.tmap_y[i]);
            }
    }
    const int MT = (T + pf::BM - 1) / pf::BM;
    const int NT = GROUPED ? out.nt_end[out.G - 1] : out.nt_end[0];  // output tiles of all layers per token tile
    const int tiles = MT * NT;
    const int KB = (K + pf::BK - 1) / pf::BK;
    // work items: (tile, k-slice), the slices of a tile on consecutive items
    const int items = tiles * ksplit;
    auto kslice = [&](int wi, int& kb0, int& kb1) {
        const int ks = wi % ksplit;
        kb0 = static_cast<int>(static_cast<long long>(KB) * ks / ksplit);
        kb1 = static_cast<int>(static_cast<long long>(KB) * (ks + 1) / ksplit);
    };

    if (threadIdx.x == 0) {
        for (int s = 0; s < Cfg::STAGES; ++s) {
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
    // inputs of this call (quantised activations) come from the preceding kernel
    asm volatile("griddepcontrol.wait;" ::: "memory");
    if (threadIdx.x == 0) SBL_TR(15, 0);  // inputs visible

    auto give_up = [&]() {
        if (!*abort_flag) {
            *abort_flag = 1;
            raise_status(status, kStatusTimeout);
        }
    };

    if (BN == 128 && warp < pf::EPI_WARPS && ksplit > 1) {
        // ------------------------------------------------------------ split-K epilogue
        // Each work item adds its int32 partial tile into the tile's slot of
        // `part` with reductions performed at L2 (no round trip), column-major
        // by token (element (t, c) of a tile at c * 128 + t, so a warp's 32
        // tokens touch 128 contiguous bytes per column).  The slots are zeroed
        // by the quantisation kernel before and dequantised by
        // split_dequant_kernel after this kernel.
        constexpr int NSL = BN / 32;
        constexpr size_t kSlot = static_cast<size_t>(pf::BM) * BN;
        const uint32_t lane_addr = static_cast<uint32_t>(warp * 32) << 16;
        int tc = 0;
        for (int wi = blockIdx.x; wi < items; wi += gridDim.x, ++tc) {
            const int tile = wi / ksplit;
            const int mt = tile / NT;
            const int b = tc & 1;
            const uint32_t aph = (tc >> 1) & 1;
            if (!warp_wait(&sm->tmem_full[b], aph, abort_flag)) { give_up(); break; }
            tc_fence_after();
            const uint32_t tbase = tmem_base + lane_addr + b * BN;
            if (mt * pf::BM + warp * 32 < T) {
                int32_t* slot = part + static_cast<size_t>(tile) * kSlot + warp * 32 + lane;
#pragma unroll 1
                for (int k = 0; k < NSL; ++k) {
                    uint32_t cur[32];
                    tmem_ld32_nowait(tbase + 32 * k, cur);
                    tmem_ld_wait();
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        asm volatile("red.relaxed.gpu.global.add.s32 [%0], %1;" ::"l"(slot + (32 * k + i) * pf::BM),
                                     "r"(cur[i])
                                     : "memory");
                }
            }
            tc_fence_before();
            mbar_arrive(&sm->tmem_empty[b]);  // the accumulator buffer is free for the MMA
        }
    } else if (warp < pf::EPI_WARPS) {
        // ------------------------------------------------------------ epilogue
        // Warp w owns TMEM lanes 32w .. 32w + 31 (32 tokens of the tile).  Per
        // tile it first copies the tile's row scales into its own shared-memory
        // slice (before waiting for the accumulator), then walks the 32-column
        // TMEM slices with the next slice's load in flight while the current one
        // is dequantised.  Every 128 output bytes per token (a "round": 32 fp32
        // or 64 bf16 columns) go into one of the warp's two 128B-swizzled
        // 32-row staging boxes and out by one TMA store, which writes whole
        // lines and clips the ragged edges.  Nothing synchronises beyond the warp.
        auto run = [&](auto bf16_tag) {
            constexpr bool BF = decltype(bf16_tag)::value;
            constexpr int SPR = BF ? 2 : 1;          // 32-column slices per round
            constexpr int NSL = BN / 32;             // slices per tile
            const int row = warp * 32 + lane;        // TMEM lane == token within the tile
            const uint32_t lane_addr = static_cast<uint32_t>(warp * 32) << 16;
            float* const wsc = sm->wscale[warp];
            int tc = 0;
            int ep_round = 0;
            uint32_t nstore = 0;
            for (int tile = blockIdx.x; tile < tiles; tile += gridDim.x, ++tc) {
                const int mt = tile / NT;  // output tiles fastest: a token tile is read once
                int g = 0, nt = tile % NT;
                if (GROUPED) {
                    while (g + 1 < out.G && nt >= out.nt_end[g]) ++g;
                    if (g > 0) nt -= out.nt_end[g - 1];
                }
                const int O = out.O[g], y_vec = out.y_vec[g];
                const float* const row_scale = out.row_scale[g];
                const int b = tc & 1;
                const uint32_t aph = (tc >> 1) & 1;
                __syncwarp();
#pragma unroll
                for (int k = 0; k < NSL; ++k) {
                    const int o = nt * BN + 32 * k + lane;
                    wsc[32 * k + lane] = o < O ? __ldg(row_scale + o) : 0.f;
                }
                __syncwarp();
                // warp-uniform decision: tcgen05.ld below is a .sync.aligned warp instruction
                if (!warp_wait(&sm->tmem_full[b], aph, abort_flag)) { give_up(); break; }
                if (threadIdx.x == 0) SBL_TR(6, tc);
                tc_fence_after();
                const int t = mt * pf::BM + row;
                const bool tvalid = t < T;
                const float inv_s = tvalid ? __frcp_rn(s_tok[t]) : 0.f;
                const uint32_t tbase = tmem_base + lane_addr + b * BN;
                uint32_t ra[32], rb[32];
                uint32_t q[32];
                // one 32-column slice k (H = k % SPR): convert `cur` while slice k + 1 loads into `nxt`
                auto slice = [&](auto h_tag, const int k, uint32_t (&cur)[32], uint32_t (&nxt)[32]) {
                    constexpr int H = decltype(h_tag)::value;
                    const bool more = k + 1 < NSL;
                    if (more) {
                        tmem_ld32_nowait(tbase + 32 * (k + 1), nxt);
                    } else {
                        tc_fence_before();
                        mbar_arrive(&sm->tmem_empty[b]);  // the accumulator buffer is free for the MMA
                    }
                    if (H == 0 && threadIdx.x == 0) SBL_TR(10, ep_round);
                    const float* sc = wsc + 32 * k;
#pragma unroll
                    for (int i = 0; i < 32; i += 4) {
                        const float4 s4 = *reinterpret_cast<const float4*>(sc + i);
                        const float f0 = __fmul_rn(__fmul_rn(static_cast<float>(static_cast<int>(cur[i + 0])), s4.x), inv_s);
                        const float f1 = __fmul_rn(__fmul_rn(static_cast<float>(static_cast<int>(cur[i + 1])), s4.y), inv_s);
                        const float f2 = __fmul_rn(__fmul_rn(static_cast<float>(static_cast<int>(cur[i + 2])), s4.z), inv_s);
                        const float f3 = __fmul_rn(__fmul_rn(static_cast<float>(static_cast<int>(cur[i + 3])), s4.w), inv_s);
                        if (BF) {
                            const __nv_bfloat162 h01 = __floats2bfloat162_rn(f0, f1);
                            const __nv_bfloat162 h23 = __floats2bfloat162_rn(f2, f3);
                            q[16 * H + i / 2] = *reinterpret_cast<const uint32_t*>(&h01);
                            q[16 * H + i / 2 + 1] = *reinterpret_cast<const uint32_t*>(&h23);
                        } else {
                            q[i] = __float_as_uint(f0);
                            q[i + 1] = __float_as_uint(f1);
                            q[i + 2] = __float_as_uint(f2);
                            q[i + 3] = __float_as_uint(f3);
                        }
                    }
                    int32_t* const acc_out = out.acc_out[g];
                    if (acc_out && tvalid) {
                        const long long base = static_cast<long long>(t) * O + nt * BN + 32 * k;
#pragma unroll
                        for (int i = 0; i < 32; ++i)
                            if (nt * BN + 32 * k + i < O) acc_out[base + i] = static_cast<int>(cur[i]);
                    }
                    if (H == SPR - 1) {
                        const int o0 = nt * BN + 32 * (k - H);
                        if (threadIdx.x == 0) SBL_TR(11, ep_round);
                        if (y_vec) {
                            uint8_t* const box = sm->ystage[warp][nstore & 1];
                            if (lane == 0) bulk_wait_read<1>();
                            __syncwarp();
#pragma unroll
                            for (int c = 0; c < 8; ++c) {
                                const uint32_t a = smem_u32(box + lane * 128 + ((c ^ (lane & 7)) << 4));
                                asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(a), "r"(q[4 * c]),
                                             "r"(q[4 * c + 1]), "r"(q[4 * c + 2]), "r"(q[4 * c + 3])
                                             : "memory");
                            }
                            fence_proxy_async_smem();
                            __syncwarp();
                            if (lane == 0) tma_store_2d(tile_owner<GROUPED>(out, tile % NT).tmap_y, smem_u32(box), o0, mt * pf::BM + warp * 32);
                            ++nstore;
                        } else if (tvalid) {
                            // direct stores: shapes whose row pitch is not a multiple of 16 bytes
                            void* const y = out.y[g];
                            const long long base = static_cast<long long>(t) * O + o0;
#pragma unroll
                            for (int i = 0; i < 32; ++i) {
                                if (BF) {
                                    if (o0 + 2 * i < O)
                                        reinterpret_cast<uint16_t*>(y)[base + 2 * i] = static_cast<uint16_t>(q[i] & 0xFFFFu);
                                    if (o0 + 2 * i + 1 < O)
                                        reinterpret_cast<uint16_t*>(y)[base + 2 * i + 1] = static_cast<uint16_t>(q[i] >> 16);
                                } else if (o0 + i < O) {
                                    reinterpret_cast<uint32_t*>(y)[base + i] = q[i];
                                }
                            }
                        }
                        ++ep_round;
                    }
                    if (more) tmem_ld_wait();
                };
                tmem_ld32_nowait(tbase, ra);
                tmem_ld_wait();
                for (int k = 0; k < NSL; k += 2) {
                    if (SPR == 2) {
                        slice(std::integral_constant<int, 0>{}, k, ra, rb);
                        slice(std::integral_constant<int, 1>{}, k + 1, rb, ra);
                    } else {
                        slice(std::integral_constant<int, 0>{}, k, ra, rb);
                        slice(std::integral_constant<int, 0>{}, k + 1, rb, ra);
                    }
                }
                if (threadIdx.x == 0) SBL_TR(7, tc);
            }
            if (lane == 0) bulk_wait_all();
        };
        if (y_bf16) run(std::true_type{});
        else run(std::false_type{});
    } else if (warp < Cfg::WARP_TMA) {
        // ------------------------------------------------------------ weight expansion
        const int r = threadIdx.x - pf::EPI_WARPS * 32;  // row of the B tile
        uint32_t it = 0;
        bool ok = true;
        for (int wi = blockIdx.x; wi < items && ok; wi += gridDim.x) {
            int kb0, kb1;
            kslice(wi, kb0, kb1);
            for (int kb = kb0; kb < kb1; ++kb, ++it) {
                const int s = it % Cfg::STAGES;
                const uint32_t ph = (it / Cfg::STAGES) & 1;
                // the codes have landed, and the producer only issued them once the
                // MMA had released this stage, so b[s] is free as well
                if (!mbar_wait(&sm->full_tma[s], ph, abort_flag)) { give_up(); ok = false; break; }
                if (r == 0) SBL_TR(1, it);
                // code tile rows are 32 bytes, 32B-swizzled by TMA: 16-byte half q of
                // row r sits at half q ^ ((r >> 2) & 1)
                const uint8_t* src = sm->p[s] + r * 32;
                const int hs = (r >> 2) & 1;
                const uint4 p0 = *reinterpret_cast<const uint4*>(src + (hs << 4));
                const uint4 p1 = *reinterpret_cast<const uint4*>(src + ((hs ^ 1) << 4));
                uint8_t* dst = sm->b[s] + r * 128;
                const int sw = r & 7;
                const uint32_t words[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    uint32_t e[4];
                    expand_pairs(words[c], e);
                    const uint32_t a = smem_u32(dst + ((c ^ sw) << 4));
                    asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(a), "r"(e[0]), "r"(e[1]), "r"(e[2]),
                                 "r"(e[3])
                                 : "memory");
                }
                fence_proxy_async_smem();
                mbar_arrive(&sm->full_dec[s]);
                if (r == 0) SBL_TR(2, it);
            }
        }
    } else if (warp == Cfg::WARP_TMA) {
        // ------------------------------------------------------------ activation TMA producer
        if (lane == 0) {
            uint32_t it = 0;
            bool ok = true;
            for (int wi = blockIdx.x; wi < items && ok; wi += gridDim.x) {
                const int tile = wi / ksplit;
                const int mt = tile / NT;  // output tiles fastest: a token tile is read once
                const TileOwner own = tile_owner<GROUPED>(out, tile % NT);
                int kb0, kb1;
                kslice(wi, kb0, kb1);
                for (int kb = kb0; kb < kb1; ++kb, ++it) {
                    const int s = it % Cfg::STAGES;
                    const uint32_t ph = (it / Cfg::STAGES) & 1;
                    if (!mbar_wait(&sm->empty[s], ph ^ 1, abort_flag)) { give_up(); ok = false; break; }
                    SBL_TR(0, it);
                    mbar_arrive_expect_tx(&sm->full_tma[s], pf::A_BYTES + Cfg::P_BYTES);
                    tma_load_2d(smem_u32(sm->a[s]), &tmap_x, kb * pf::BK, mt * pf::BM, &sm->full_tma[s]);
                    tma_load_2d(smem_u32(sm->p[s]), own.tmap_w, kb * (pf::BK / 4), own.nt * BN, &sm->full_tma[s]);
                }
            }
            // let every issued load land before the CTA can exit
            const uint32_t first = it > Cfg::STAGES ? it - Cfg::STAGES : 0;
            volatile int never = 0;
            for (uint32_t j = first; j < it; ++j)
                if (!mbar_wait(&sm->full_tma[j % Cfg::STAGES], (j / Cfg::STAGES) & 1, &never)) give_up();
        }
    } else {
        // ------------------------------------------------------------ MMA issuer
        // Per stage: wait for the activation and expanded weight tiles, four
        // K = 32 MMAs, commit (releases the stage when the MMAs finish); per
        // tile: wait for a free accumulator buffer, commit it to the epilogue.
        if (lane == 0) {
            const uint32_t idesc = i8_idesc<pf::BM, BN>();
            uint32_t it = 0;
            int tc = 0;
            bool ok = true;
            for (int wi = blockIdx.x; wi < items && ok; wi += gridDim.x, ++tc) {
                const int b = tc & 1;
                const uint32_t aph = (tc >> 1) & 1;
                if (!mbar_wait(&sm->tmem_empty[b], aph ^ 1, abort_flag)) { give_up(); break; }
                tc_fence_after();
                const uint32_t d = tmem_base + b * BN;
                int kb0, kb1;
                kslice(wi, kb0, kb1);
                for (int kb = kb0; kb < kb1; ++kb, ++it) {
                    const int s = it % Cfg::STAGES;
                    const uint32_t ph = (it / Cfg::STAGES) & 1;
                    if (!mbar_wait(&sm->full_tma[s], ph, abort_flag) || !mbar_wait(&sm->full_dec[s], ph, abort_flag)) {
                        give_up(); ok = false; break;
                    }
                    tc_fence_after();
                    const uint32_t a0 = smem_u32(sm->a[s]), b0 = smem_u32(sm->b[s]);
#pragma unroll
                    for (int kk = 0; kk < pf::BK / 32; ++kk)
                        tc_mma(d, sw128_desc(a0 + kk * 32), sw128_desc(b0 + kk * 32), idesc, (kb != kb0) || (kk != 0));
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
    if (threadIdx.x == 0) SBL_TR(13, 0);  // every role done
    if (threadIdx.x == 0) SBL_TRB(16);
    if (warp == Cfg::WARP_MMA) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(Cfg::TMEM_COLS)
                     : "memory");
    }
}

// G layers (G <= kPrefillMaxGroup) that read the same quantised activations,
// in one launch of the one-CTA kernel.
template <int BN>
static cudaError_t launch_prefill_bn(const int8_t* xperm, const float* s_tok, long long T, long long K, int G,
                                     const uint8_t* const* packed, const float* const* row_scale, const long long* O,
                                     void* const* y, int y_bf16, int32_t* const* acc_out, int ksplit, int32_t* part,
                                     unsigned* status, int num_sms, cudaStream_t stream) {
    EncodeTiledFn enc = get_encode_fn();
    if (!enc) return cudaErrorNotSupported;
    if (G < 1 || G > kPrefillMaxGroup) return cudaErrorInvalidValue;
    CUtensorMap map_x;
    const cuuint32_t estr[2] = {1, 1};
    {
        const cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(T)};
        const cuuint64_t strides[1] = {static_cast<cuuint64_t>(K)};
        const cuuint32_t box[2] = {static_cast<cuuint32_t>(pf::BK), static_cast<cuuint32_t>(pf::BM)};
        if (enc(&map_x, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<int8_t*>(xperm), dims, strides, box, estr,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    PrefillOut out;
    memset(&out, 0, sizeof(out));
    out.G = G;
    int nt_end = 0;
    for (int g = 0; g < G; ++g) {
        {
            const cuuint64_t dims[2] = {static_cast<cuuint64_t>(K / 4), static_cast<cuuint64_t>(O[g])};
            const cuuint64_t strides[1] = {static_cast<cuuint64_t>(K / 4)};
            const cuuint32_t box[2] = {static_cast<cuuint32_t>(pf::BK / 4), static_cast<cuuint32_t>(BN)};
            if (enc(&out.tmap_w[g], CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(packed[g]), dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_32B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
                return cudaErrorInvalidValue;
        }
        // output rows go out as 16-byte vectors when the row pitch allows it
        const int esize = y_bf16 ? 2 : 4;
        out.y_vec[g] = (static_cast<long long>(O[g]) * esize) % 16 == 0 ? 1 : 0;
        out.tmap_y[g] = map_x;
        if (out.y_vec[g]) {
            const cuuint64_t dims[2] = {static_cast<cuuint64_t>(O[g]), static_cast<cuuint64_t>(T)};
            const cuuint64_t strides[1] = {static_cast<cuuint64_t>(O[g]) * esize};
            const cuuint32_t box[2] = {static_cast<cuuint32_t>(128 / esize), 32u};
            if (enc(&out.tmap_y[g], y_bf16 ? CU_TENSOR_MAP_DATA_TYPE_UINT16 : CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, y[g],
                    dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
                out.y_vec[g] = 0;
        }
        out.row_scale[g] = row_scale[g];
        out.y[g] = y[g];
        out.acc_out[g] = acc_out ? acc_out[g] : nullptr;
        out.O[g] = static_cast<int>(O[g]);
        nt_end += static_cast<int>((O[g] + BN - 1) / BN);
        out.nt_end[g] = nt_end;
    }
    constexpr size_t smem = prefill_smem_bytes<BN>();
    static bool attr_set[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64 || !attr_set[dev]) {
        cudaError_t e = cudaFuncSetAttribute(prefill_kernel<BN, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(smem));
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(prefill_kernel<BN, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     static_cast<int>(smem));
        if (e != cudaSuccess) return e;
        if (dev >= 0 && dev < 64) attr_set[dev] = true;
    }
    const long long items = ((T + pf::BM - 1) / pf::BM) * nt_end * ksplit;
    const int grid = static_cast<int>(items < num_sms ? items : num_sms);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(PrefillCfg<BN>::THREADS);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (G > 1)
        return cudaLaunchKernelEx(&cfg, prefill_kernel<BN, true>, map_x, out, s_tok, static_cast<int>(T),
                                  static_cast<int>(K), y_bf16, ksplit, part, status);
    return cudaLaunchKernelEx(&cfg, prefill_kernel<BN, false>, map_x, out, s_tok, static_cast<int>(T),
                              static_cast<int>(K), y_bf16, ksplit, part, status);
}

template <int BN>
static cudaError_t launch_prefill_bn(const int8_t* xperm, const float* s_tok, long long T, long long K,
                                     const uint8_t* packed, const float* row_scale, long long O, void* y, int y_bf16,
                                     int32_t* acc_out, int ksplit, int32_t* part, unsigned* status,
                                     int num_sms, cudaStream_t stream) {
    void* yy[1] = {y};
    int32_t* aa[1] = {acc_out};
    return launch_prefill_bn<BN>(xperm, s_tok, T, K, 1, &packed, &row_scale, &O, yy, y_bf16, aa, ksplit, part,
                                 status, num_sms, stream);
}

#ifdef SBL_TRACE
cudaError_t set_prefill_trace(void* buf) {
    unsigned long long* p = static_cast<unsigned long long*>(buf);
    return cudaMemcpyToSymbol(g_trace, &p, sizeof(p));
}
#endif

int prefill_pair_clusters(cudaStream_t stream);
cudaError_t launch_prefill_pair_group(const int8_t* xperm, const float* s_tok, long long T, long long K, int G,
                                      const uint8_t* const* packed, const float* const* row_scale,
                                      const long long* O, void* const* y, int y_bf16, int32_t* const* acc_out,
                                      unsigned* status, cudaStream_t stream);
cudaError_t launch_prefill_pair(const int8_t* xperm, const float* s_tok, long long T, long long K,
                                const uint8_t* packed, const float* row_scale, long long O, void* y, int y_bf16,
                                int32_t* acc_out, unsigned* status, cudaStream_t stream);

// The dense tensor-core kernel the automatic choice takes: 0 one CTA with
// 128-output tiles, 1 one CTA with 256-output tiles, 2 CTA pairs.
// Cost model in units of one 128 x 256 tile on one SM: waves of tiles times
// the time of one tile.  A narrow 128 x 128 tile costs about 0.65 of a wide
// one (BN = 256 halves the activation traffic and MMA issue overhead per
// output); a CTA pair finishes its 256 x 256 tile in about kPairCost of a wide
// one-CTA tile (half the expansion and shared-memory traffic per SM).
int choose_dense_prefill(long long T, long long O, int num_sms, cudaStream_t stream) {
    constexpr double kNarrowCost = 0.65, kPairCost = 0.65;
    const long long mt = (T + pf::BM - 1) / pf::BM;
    const double wide = static_cast<double>((mt * ((O + 255) / 256) + num_sms - 1) / num_sms);
    const double narrow = kNarrowCost * static_cast<double>((mt * ((O + 127) / 128) + num_sms - 1) / num_sms);
    const int clusters = prefill_pair_clusters(stream);
    if (clusters > 0) {
        const long long pt = ((T + 255) / 256) * ((O + 255) / 256);
        if (kPairCost * static_cast<double>((pt + clusters - 1) / clusters) < (wide < narrow ? wide : narrow)) return 2;
    }
    return wide <= narrow ? 1 : 0;
}

// Dequantisation of split-K accumulators: y[t, o] = acc[t, o] * row_scale[o] *
// (1 / s_tok[t]), the float steps of the one-CTA epilogue.  A block of 8 warps
// takes 32 tokens x 32 outputs: it reads the column-major slots with lanes
// along tokens, transposes through shared memory and writes output rows with
// lanes along outputs.  A programmatic dependent of the contraction kernel.
__global__ void __launch_bounds__(256) split_dequant_kernel(const int32_t* __restrict__ part,
                                                            const float* __restrict__ row_scale,
                                                            const float* __restrict__ s_tok, int T, int O,
                                                            void* __restrict__ y, int y_bf16,
                                                            int32_t* __restrict__ acc_out) {
    __shared__ int box[32][33];
    asm volatile("griddepcontrol.launch_dependents;");
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int lane = threadIdx.x & 31, wy = threadIdx.x >> 5;
    const int o0 = blockIdx.x * 32, t0 = blockIdx.y * 32;
    const int NT = (O + 127) / 128;
    const int t = t0 + lane;
#pragma unroll
    for (int j = wy; j < 32; j += 8) {
        const int o = o0 + j;
        int v = 0;
        if (t < T && o < O) {
            const size_t tile = static_cast<size_t>(t / pf::BM) * NT + o / 128;
            v = __ldcg(part + tile * (pf::BM * 128) + (o % 128) * pf::BM + (t % pf::BM));
        }
        box[j][lane] = v;
    }
    __syncthreads();
    const int o = o0 + lane;
    if (o >= O) return;
    const float sc = __ldg(row_scale + o);
#pragma unroll
    for (int r = wy; r < 32; r += 8) {
        const int tt = t0 + r;
        if (tt >= T) break;
        const int a = box[lane][r];
        const float f = __fmul_rn(__fmul_rn(static_cast<float>(a), sc), __frcp_rn(s_tok[tt]));
        const size_t idx = static_cast<size_t>(tt) * O + o;
        if (y_bf16)
            reinterpret_cast<__nv_bfloat16_raw*>(y)[idx] = static_cast<__nv_bfloat16_raw>(__float2bfloat16_rn(f));
        else
            reinterpret_cast<float*>(y)[idx] = f;
        if (acc_out) acc_out[idx] = a;
    }
}

// Split-K plan of the one-CTA kernel with 128-output tiles: when its tiles
// fill at most half of the SMs, each tile's k-blocks are divided among up to
// num_sms / tiles CTAs (at most 16, at least two k-blocks each).  Measured on
// B200, a split costs about as much as 8 to 10 k-blocks of one CTA (L2
// reductions and the dequantisation kernel), so it is taken only when it
// removes at least 12 k-blocks from each CTA's run.  Returns the number of
// slices (1: no split).
int prefill_ksplit(long long T, long long K, long long O, int num_sms) {
    const long long tiles = ((T + pf::BM - 1) / pf::BM) * ((O + 127) / 128);
    const long long kb = (K + pf::BK - 1) / pf::BK;
    if (tiles * 2 > num_sms || kb < 4) return 1;
    long long ks = num_sms / tiles;
    if (ks > kb / 2) ks = kb / 2;
    if (ks > 16) ks = 16;
    if (ks < 2 || kb - (kb + ks - 1) / ks < 12) return 1;
    return static_cast<int>(ks);
}

// Workspace of a split: one int32 accumulator tile (128 tokens x 128 outputs)
// per tile, zero when the contraction kernel starts.
size_t prefill_split_part_bytes(long long T, long long O, int ksplit) {
    const size_t tiles = static_cast<size_t>((T + pf::BM - 1) / pf::BM) * ((O + 127) / 128);
    return ksplit > 1 ? tiles * pf::BM * 128 * 4 : 0;
}

cudaError_t launch_prefill(const int8_t* xperm, const float* s_tok, long long T, long long K, const uint8_t* packed,
                           const float* row_scale, long long O, void* y, int y_bf16, int32_t* acc_out,
                           unsigned* status, int num_sms, int variant, int ksplit, int32_t* part,
                           cudaStream_t stream) {
    // variant 0: the automatic choice; 1: one CTA (BN by wave count); 2: CTA pairs.
    // ksplit > 1 (not with CTA pairs): the one-CTA kernel with 128-output tiles,
    // split along k into `part` (zero on entry), then split_dequant_kernel.
    if (ksplit > 1 && variant != 2) {
        cudaError_t e = launch_prefill_bn<128>(xperm, s_tok, T, K, packed, row_scale, O, y, y_bf16, acc_out, ksplit,
                                               part, status, num_sms, stream);
        if (e != cudaSuccess) return e;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(static_cast<unsigned>((O + 31) / 32), static_cast<unsigned>((T + 31) / 32));
        cfg.blockDim = dim3(256);
        cfg.stream = stream;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        return cudaLaunchKernelEx(&cfg, split_dequant_kernel, static_cast<const int32_t*>(part), row_scale, s_tok,
                                  static_cast<int>(T), static_cast<int>(O), y, y_bf16, acc_out);
    }
    int kind;
    if (variant == 2) {
        kind = 2;
    } else {
        kind = choose_dense_prefill(T, O, num_sms, stream);
        if (variant == 1 && kind == 2) {
            const long long mt = (T + pf::BM - 1) / pf::BM;
            const double wide = static_cast<double>((mt * ((O + 255) / 256) + num_sms - 1) / num_sms);
            const double narrow = 0.65 * static_cast<double>((mt * ((O + 127) / 128) + num_sms - 1) / num_sms);
            kind = wide <= narrow ? 1 : 0;
        }
    }
    if (kind == 2)
        return launch_prefill_pair(xperm, s_tok, T, K, packed, row_scale, O, y, y_bf16, acc_out, status, stream);
    if (kind == 1)
        return launch_prefill_bn<256>(xperm, s_tok, T, K, packed, row_scale, O, y, y_bf16, acc_out, 1, nullptr,
                                      status, num_sms, stream);
    return launch_prefill_bn<128>(xperm, s_tok, T, K, packed, row_scale, O, y, y_bf16, acc_out, 1, nullptr, status,
                                  num_sms, stream);
}

// G layers (1 <= G <= prefill_max_group()) that read the same quantised
// activations in one launch: their output tiles are scheduled together on
// the kernel the cost model of choose_dense_prefill picks for the sum of
// their tiles (CTA pairs, or one CTA with 256- or 128-output tiles; the split
// along k is not used).
int prefill_max_group() { return kPrefillMaxGroup; }

cudaError_t launch_prefill_grouped(const int8_t* xperm, const float* s_tok, long long T, long long K, int G,
                                   const uint8_t* const* packed, const float* const* row_scale, const long long* O,
                                   void* const* y, int y_bf16, int32_t* const* acc_out, unsigned* status,
                                   int num_sms, cudaStream_t stream) {
    constexpr double kNarrowCost = 0.65, kPairCost = 0.65;
    const long long mt = (T + pf::BM - 1) / pf::BM;
    long long t256 = 0, t128 = 0;
    for (int g = 0; g < G; ++g) {
        t256 += (O[g] + 255) / 256;
        t128 += (O[g] + 127) / 128;
    }
    const double wide = static_cast<double>((mt * t256 + num_sms - 1) / num_sms);
    const double narrow = kNarrowCost * static_cast<double>((mt * t128 + num_sms - 1) / num_sms);
    const int clusters = prefill_pair_clusters(stream);
    if (clusters > 0) {
        const long long pt = ((T + 255) / 256) * t256;
        if (kPairCost * static_cast<double>((pt + clusters - 1) / clusters) < (wide < narrow ? wide : narrow))
            return launch_prefill_pair_group(xperm, s_tok, T, K, G, packed, row_scale, O, y, y_bf16, acc_out, status,
                                             stream);
    }
    if (wide <= narrow)
        return launch_prefill_bn<256>(xperm, s_tok, T, K, G, packed, row_scale, O, y, y_bf16, acc_out, 1, nullptr,
                                      status, num_sms, stream);
    return launch_prefill_bn<128>(xperm, s_tok, T, K, G, packed, row_scale, O, y, y_bf16, acc_out, 1, nullptr, status,
                                  num_sms, stream);
}

}  // namespace sbl
