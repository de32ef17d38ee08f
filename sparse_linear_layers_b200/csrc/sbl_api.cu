// C ABI of the Sparse-BitLinear library: argument validation, workspace
// layout, path dispatch and the per-device status word.  All arithmetic runs
// in the kernels of prep.cu, quant.cu, decode.cu, decode_mma.cu, prefill.cu, prefill_pair.cu, prefill_sp.cu,
// mask_monitor.cu, backward.cu and backward_tc.cu.
#include <cstdint>
#include <cstdio>
#include <cuda_runtime.h>

#include "sbl.h"
#include "sbl_common.cuh"

namespace sbl {
cudaError_t launch_prep(const float* W, long long O, long long K, int n, int m, uint8_t* packed, float* row_scale,
                        uint8_t* mask_bits, int scale_bf16, int scale_global, unsigned* status,
                        cudaStream_t stream);
int prep_max_group();
cudaError_t launch_prep_grouped(int G, const float* const* W, const long long* O, long long K, int n, int m,
                                uint8_t* const* packed, float* const* row_scale, uint8_t* const* mask_bits,
                                unsigned* status, cudaStream_t stream);
cudaError_t launch_quant(const uint16_t* x, long long T, long long K, int8_t* xq, float* s_tok, int layout,
                         unsigned* status, cudaStream_t stream, void* zero16 = nullptr, long long nzero16 = 0);
constexpr int kLayoutNatural = 0, kLayoutPairs = 1;
cudaError_t launch_decode(const uint8_t* packed, const float* row_scale, long long O, long long K,
                          const uint16_t* x, long long T, void* y, int y_bf16, int32_t* acc_out, unsigned* status,
                          int num_sms, cudaStream_t stream);
bool decode_mma_supported(long long K);
cudaError_t launch_decode_mma(const uint8_t* packed, const float* row_scale, long long O, long long K,
                              const uint16_t* x, long long T, void* y, int y_bf16, int32_t* acc_out, unsigned* status,
                              int num_sms, cudaStream_t stream, const int8_t* xq_in = nullptr,
                              const float* stok_in = nullptr);
cudaError_t launch_rmsnorm_quant(const uint16_t* x, const float* g, float eps, long long T, long long K, int8_t* xq,
                                 float* s_tok, int layout, unsigned* status, cudaStream_t stream, void* zero16,
                                 long long nzero16);
cudaError_t launch_mask_monitor(const uint8_t* old_bits, const uint8_t* new_bits, long long O, long long K, int n,
                                int m, unsigned long long* totals, uint32_t* row_changed, cudaStream_t stream);
long long ste_backward_tiles(long long rows, long long K);
cudaError_t launch_ste_backward(const float* dY, long long T, long long O, long long K, const uint8_t* packed,
                                const float* row_scale, const int8_t* xq, const float* s_tok, float* dX, float* dW,
                                int dw_ternary, cudaStream_t stream);
int decode_max_group();
int prefill_max_group();
cudaError_t launch_prefill_grouped(const int8_t* xperm, const float* s_tok, long long T, long long K, int G,
                                   const uint8_t* const* packed, const float* const* row_scale, const long long* O,
                                   void* const* y, int y_bf16, int32_t* const* acc_out, unsigned* status,
                                   int num_sms, cudaStream_t stream);
cudaError_t launch_decode_grouped(int G, const uint8_t* const* packed, const float* const* row_scale,
                                  const long long* O, long long K, const uint16_t* x, long long T, void* const* y,
                                  int y_bf16, int32_t* const* acc_out, unsigned* status, int num_sms,
                                  cudaStream_t stream);
size_t backward_tc_workspace_bytes(long long T, long long O, long long K, int need_dx, int need_dw);
cudaError_t launch_backward_tc(const float* dY, long long T, long long O, const int8_t* xq, const float* s_tok,
                               long long K, const uint8_t* packed, const float* row_scale, float* dX, float* dW,
                               int dw_ternary, void* ws, unsigned* status, int num_sms, cudaStream_t stream);
cudaError_t launch_prefill(const int8_t* xperm, const float* s_tok, long long T, long long K, const uint8_t* packed,
                           const float* row_scale, long long O, void* y, int y_bf16, int32_t* acc_out,
                           unsigned* status, int num_sms, int variant, int ksplit, int32_t* part,
                           cudaStream_t stream);
constexpr int kPrefillAuto = 0, kPrefillOneCta = 1, kPrefillPair = 2;
int prefill_ksplit(long long T, long long K, long long O, int num_sms);
size_t prefill_split_part_bytes(long long T, long long O, int ksplit);
int choose_dense_prefill(long long T, long long O, int num_sms, cudaStream_t stream);
size_t sp_scratch_bytes(long long O, long long K);
cudaError_t launch_xq_to_pairs(const int8_t* xq, long long T, long long K, int8_t* out, int num_sms,
                               cudaStream_t stream);
cudaError_t launch_prefill_sp(const int8_t* xq, const float* s_tok, long long T, long long K, const uint8_t* packed,
                              const float* row_scale, long long O, void* y, int y_bf16, int32_t* acc_out,
                              uint8_t* scratch, unsigned* status, int num_sms, cudaStream_t stream);
#ifdef SBL_TRACE
cudaError_t set_prefill_trace(void* buf);
cudaError_t set_pair_trace(void* buf);
#endif

// Status word: one per device, read and cleared by sbl_device_status().
__device__ unsigned g_status_word;

__global__ void bounded_wait_selftest(uint32_t max_polls, unsigned* status) {
    __shared__ uint64_t bar;
    if (threadIdx.x != 0) return;
    mbar_init(&bar, 1);
    fence_barrier_init();
    for (uint32_t i = 0; i < max_polls; ++i)
        if (mbar_try_wait(&bar, 0)) return;  // nothing ever arrives: phase 0 never completes
    raise_status(status, kStatusTimeout);
}
}  // namespace sbl

namespace {

constexpr int kMaxDevices = 64;
constexpr long long kMaxK = 1ll << 24;            // keeps |acc| <= 127 * K below 2^31
constexpr long long kDecodeMaxTokens = 16;
constexpr long long kDecodeMaxK = 24576;          // decode holds 8 tokens x K int8 in shared memory
constexpr long long kDecodeMmaMinTokens = 3;      // from here on the decode runs on the warp-level MMA

struct DeviceInfo {
    unsigned* status = nullptr;
    int num_sms = 0;
};
DeviceInfo g_dev[kMaxDevices];

sbl_status device_info(DeviceInfo** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return SBL_ERR_CUDA;
    DeviceInfo& d = g_dev[dev];
    if (!d.status) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, sbl::g_status_word) != cudaSuccess) return SBL_ERR_CUDA;
        int sms = 0;
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return SBL_ERR_CUDA;
        d.num_sms = sms;
        d.status = static_cast<unsigned*>(p);
    }
    *out = &d;
    return SBL_OK;
}

inline bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

// 2:4, 3:4 and 6:8 (the patterns of the guide and the halo card) and 4:8 (the
// guide's "Architectural Comparison" table)
inline bool nm_ok(int n, int m) {
    return (n == 2 && m == 4) || (n == 3 && m == 4) || (n == 6 && m == 8) || (n == 4 && m == 8);
}

inline size_t round256(size_t b) { return (b + 255) & ~static_cast<size_t>(255); }

inline sbl_status from_cuda(cudaError_t e) { return e == cudaSuccess ? SBL_OK : SBL_ERR_CUDA; }

sbl_status check_k(long long K) {
    if (K <= 0 || K % 16 != 0) return SBL_ERR_INVALID_ARG;
    if (K > kMaxK) return SBL_ERR_UNSUPPORTED;
    return SBL_OK;
}

}  // namespace

extern "C" {

sbl_status sbl_prepare_weights(const float* W, int64_t O, int64_t K, int n, int m, uint8_t* packed,
                               float* row_scale, uint8_t* mask_bits, void* stream) {
    return sbl_prepare_weights_ex(W, O, K, n, m, packed, row_scale, mask_bits, 0, stream);
}

sbl_status sbl_prepare_weights_ex(const float* W, int64_t O, int64_t K, int n, int m, uint8_t* packed,
                                  float* row_scale, uint8_t* mask_bits, int flags, void* stream) {
    if (O < 0) return SBL_ERR_INVALID_ARG;
    if (flags & ~(SBL_PREP_SCALE_BF16 | SBL_PREP_SCALE_GLOBAL)) return SBL_ERR_INVALID_ARG;
    if ((flags & SBL_PREP_SCALE_GLOBAL) && O * K >= (1ll << 32)) return SBL_ERR_UNSUPPORTED;
    if (sbl_status s = check_k(K)) return s;
    if (!nm_ok(n, m)) return SBL_ERR_UNSUPPORTED;
    if (O == 0) return SBL_OK;
    if (!W || !packed || !row_scale) return SBL_ERR_INVALID_ARG;
    if (!aligned(W, 16) || !aligned(packed, 16) || !aligned(row_scale, 16)) return SBL_ERR_INVALID_ARG;
    if (mask_bits && !aligned(mask_bits, 16)) return SBL_ERR_INVALID_ARG;
    if (O > (1ll << 31) - 1) return SBL_ERR_UNSUPPORTED;
    DeviceInfo* d;
    if (sbl_status s = device_info(&d)) return s;
    return from_cuda(sbl::launch_prep(W, O, K, n, m, packed, row_scale, mask_bits,
                                      (flags & SBL_PREP_SCALE_BF16) ? 1 : 0, (flags & SBL_PREP_SCALE_GLOBAL) ? 1 : 0,
                                      d->status,
                                      static_cast<cudaStream_t>(stream)));
}

sbl_status sbl_prepare_weights_grouped(int G, const float* const* W, const int64_t* O, int64_t K, int n, int m,
                                       uint8_t* const* packed, float* const* row_scale, uint8_t* const* mask_bits,
                                       void* stream) {
    if (G < 1 || G > SBL_MAX_GROUP || G > sbl::prep_max_group() || !W || !O || !packed || !row_scale)
        return SBL_ERR_INVALID_ARG;
    if (sbl_status s = check_k(K)) return s;
    if (!nm_ok(n, m)) return SBL_ERR_UNSUPPORTED;
    long long rows = 0, Ol[SBL_MAX_GROUP];
    for (int g = 0; g < G; ++g) {
        if (O[g] < 0 || O[g] > (1ll << 31) - 1) return SBL_ERR_INVALID_ARG;
        Ol[g] = O[g];
        rows += O[g];
        if (O[g] == 0) continue;
        if (!W[g] || !packed[g] || !row_scale[g]) return SBL_ERR_INVALID_ARG;
        if (!aligned(W[g], 16) || !aligned(packed[g], 16) || !aligned(row_scale[g], 16)) return SBL_ERR_INVALID_ARG;
        if (mask_bits && mask_bits[g] && !aligned(mask_bits[g], 16)) return SBL_ERR_INVALID_ARG;
    }
    if (rows == 0) return SBL_OK;
    if (rows > (1ll << 31) - 1) return SBL_ERR_UNSUPPORTED;
    DeviceInfo* d;
    if (sbl_status s = device_info(&d)) return s;
    return from_cuda(sbl::launch_prep_grouped(G, W, Ol, K, n, m, packed, row_scale, mask_bits, d->status,
                                              static_cast<cudaStream_t>(stream)));
}

sbl_status sbl_quant_act(const uint16_t* x_bf16, int64_t T, int64_t K, int8_t* x_q, float* s_tok, void* stream) {
    if (T < 0) return SBL_ERR_INVALID_ARG;
    if (sbl_status s = check_k(K)) return s;
    if (T == 0) return SBL_OK;
    if (!x_bf16 || !x_q || !s_tok) return SBL_ERR_INVALID_ARG;
    if (!aligned(x_bf16, 16) || !aligned(x_q, 16) || !aligned(s_tok, 16)) return SBL_ERR_INVALID_ARG;
    if (T > (1ll << 31) - 1) return SBL_ERR_UNSUPPORTED;
    DeviceInfo* d;
    if (sbl_status s = device_info(&d)) return s;
    return from_cuda(sbl::launch_quant(x_bf16, T, K, x_q, s_tok, sbl::kLayoutNatural, d->status,
                                       static_cast<cudaStream_t>(stream)));
}

sbl_status sbl_rmsnorm_quant_act(const uint16_t* x_bf16, const float* g, float eps, int64_t T, int64_t K,
                                 int8_t* x_q, float* s_tok, void* stream) {
    if (T < 0) return SBL_ERR_INVALID_ARG;
    if (sbl_status s = check_k(K)) return s;
    if (!(eps >= 0.0f) || !(eps < 3.0e38f)) return SBL_ERR_INVALID_ARG;
    if (T == 0) return SBL_OK;
    if (!x_bf16 || !g || !x_q || !s_tok) return SBL_ERR_INVALID_ARG;
    if (!aligned(x_bf16, 16) || !aligned(g, 16) || !aligned(x_q, 16) || !aligned(s_tok, 16))
        return SBL_ERR_INVALID_ARG;
    if (T > (1ll << 31) - 1) return SBL_ERR_UNSUPPORTED;
    DeviceInfo* d;
    if (sbl_status s = device_info(&d)) return s;
    return from_cuda(sbl::launch_rmsnorm_quant(x_bf16, g, eps, T, K, x_q, s_tok, sbl::kLayoutNatural, d->status,
                                               static_cast<cudaStream_t>(stream), nullptr, 0));
}

sbl_status sbl_mask_monitor(const uint8_t* old_bits, const uint8_t* new_bits, int64_t O, int64_t K, int n, int m,
                            uint64_t* totals, uint32_t* row_changed, void* stream) {
    if (O < 0) return SBL_ERR_INVALID_ARG;
    if (sbl_status s = check_k(K)) return s;
    if (!nm_ok(n, m)) return SBL_ERR_UNSUPPORTED;
    if (!totals || !aligned(totals, 8)) return SBL_ERR_INVALID_ARG;
    if (O > 0 && (!old_bits || !new_bits || !aligned(old_bits, 16) || !aligned(new_bits, 16))) return SBL_ERR_INVALID_ARG;
    if (row_changed && !aligned(row_changed, 4)) return SBL_ERR_INVALID_ARG;
    if (O > (1ll << 31) - 1) return SBL_ERR_UNSUPPORTED;
    DeviceInfo* d;
    if (sbl_status s = device_info(&d)) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (O == 0) return from_cuda(cudaMemsetAsync(totals, 0, 2 * sizeof(uint64_t), st));
    return from_cuda(sbl::launch_mask_monitor(old_bits, new_bits, O, K, n, m,
                                              reinterpret_cast<unsigned long long*>(totals), row_changed, st));
}

sbl_status sbl_linear_backward(const float* dY, int64_t T, int64_t O, const int8_t* x_q, const float* s_tok,
                               int64_t K, const uint8_t* packed, const float* row_scale, float* dX, float* dW,
                               int flags, void* stream) {
    if (T < 0 || O < 0) return SBL_ERR_INVALID_ARG;
    if (flags & ~SBL_BWD_DW_TERNARY) return SBL_ERR_INVALID_ARG;
    if (sbl_status s = check_k(K)) return s;
    if (!dX && !dW) return SBL_ERR_INVALID_ARG;
    const bool any_dx = dX && T > 0, any_dw = dW && O > 0;  // outputs with elements
    const bool ternary = (flags & SBL_BWD_DW_TERNARY) != 0;
    // what the requested outputs read: every pointer non-null and 16-byte aligned
    auto ok = [](const void* p) { return p != nullptr && aligned(p, 16); };
    if (any_dx && !(ok(dX) && (O == 0 || (ok(dY) && ok(packed) && ok(row_scale))))) return SBL_ERR_INVALID_ARG;
    if (any_dw && !(ok(dW) && (T == 0 || (ok(dY) && ok(x_q) && ok(s_tok))) && (!ternary || ok(row_scale))))
        return SBL_ERR_INVALID_ARG;
    if (sbl::ste_backward_tiles(T, K) > (1ll << 31) - 1 || sbl::ste_backward_tiles(O, K) > (1ll << 31) - 1)
        return SBL_ERR_UNSUPPORTED;
    if (!any_dx && !any_dw) return SBL_OK;
    DeviceInfo* d;
    if (sbl_status s = device_info(&d)) return s;
    return from_cuda(sbl::launch_ste_backward(dY, T, O, K, packed, row_scale, x_q, s_tok, any_dx ? dX : nullptr,
                                              any_dw ? dW : nullptr, ternary ? 1 : 0,
                                              static_cast<cudaStream_t>(stream)));
}

// Largest T and O of the tensor-core backward (grid extents of its operand passes).
constexpr long long kBwdTcMaxRows = 1ll << 21;

size_t sbl_linear_backward_workspace_bytes(int64_t T, int64_t O, int64_t K, int need_dx, int need_dw) {
    if (T < 0 || O < 0 || K <= 0) return 0;
    return sbl::backward_tc_workspace_bytes(T, O, K, need_dx ? 1 : 0, need_dw ? 1 : 0);
}

sbl_status sbl_linear_backward_ws(const float* dY, int64_t T, int64_t O, const int8_t* x_q, const float* s_tok,
                                  int64_t K, const uint8_t* packed, const float* row_scale, float* dX, float* dW,
                                  int flags, void* workspace, size_t workspace_bytes, void* stream) {
    if (T < 0 || O < 0) return SBL_ERR_INVALID_ARG;
    if (flags & ~SBL_BWD_DW_TERNARY) return SBL_ERR_INVALID_ARG;
    if (sbl_status s = check_k(K)) return s;
    if (!dX && !dW) return SBL_ERR_INVALID_ARG;
    // empty reductions (all zeros) and empty outputs: the CUDA-core entry point
    if (T == 0 || O == 0)
        return sbl_linear_backward(dY, T, O, x_q, s_tok, K, packed, row_scale, dX, dW, flags, stream);
    const bool ternary = (flags & SBL_BWD_DW_TERNARY) != 0;
    auto ok = [](const void* p) { return p != nullptr && aligned(p, 16); };
    if (dX && !(ok(dX) && ok(dY) && ok(packed) && ok(row_scale))) return SBL_ERR_INVALID_ARG;
    if (dW && !(ok(dW) && ok(dY) && ok(x_q) && ok(s_tok) && (!ternary || ok(row_scale)))) return SBL_ERR_INVALID_ARG;
    if (T > kBwdTcMaxRows || O > kBwdTcMaxRows) return SBL_ERR_UNSUPPORTED;
    const size_t need = sbl::backward_tc_workspace_bytes(T, O, K, dX != nullptr, dW != nullptr);
    if (!workspace || !aligned(workspace, 256) || workspace_bytes < need) return SBL_ERR_WORKSPACE;
    DeviceInfo* d;
    if (sbl_status s = device_info(&d)) return s;
    return from_cuda(sbl::launch_backward_tc(dY, T, O, x_q, s_tok, K, packed, row_scale, dX, dW, ternary ? 1 : 0,
                                             workspace, d->status, d->num_sms, static_cast<cudaStream_t>(stream)));
}

// Quantised activations and their scales: what every path needs.
static size_t base_workspace_bytes(int64_t T, int64_t K) {
    return round256(static_cast<size_t>(T) * static_cast<size_t>(K)) + round256(static_cast<size_t>(T) * 4);
}

// 2:4 weights on the sparse tensor cores also need their compressed form.
static bool sparse_eligible(int64_t K, int n, int m) { return n == 2 && m == 4 && K % 64 == 0; }

// Split-K area of the one-CTA prefill (one int32 accumulator tile per output
// tile); 0 when the sizes take no split.
static size_t split_bytes(int64_t T, int64_t K, int64_t O, int num_sms, int* ksplit = nullptr) {
    const int ks = sbl::prefill_ksplit(T, K, O, num_sms);
    if (ksplit) *ksplit = ks;
    if (ks <= 1) return 0;
    return sbl::prefill_split_part_bytes(T, O, ks);
}

size_t sbl_linear_workspace_bytes(int64_t T, int64_t K, int64_t O, int n, int m) {
    if (T <= 0 || K <= 0) return 0;
    size_t b = base_workspace_bytes(T, K);
    const bool prefill_sized = T > kDecodeMaxTokens || K > kDecodeMaxK;
    if (O > 0 && prefill_sized && K % 64 == 0) {
        size_t extra = sparse_eligible(K, n, m) ? sbl::sp_scratch_bytes(O, K) : 0;
        DeviceInfo* d;
        if (device_info(&d) == SBL_OK) {
            const size_t sb = split_bytes(T, K, O, d->num_sms);
            if (sb > extra) extra = sb;
        }
        b += extra;
    }
    return b;
}

// Whether the automatic choice sends a 2:4 prefill to the sparse tensor cores.
// Measured on B200 (bf16 output): at T = 32768 the sparse kernel matches or
// beats the dense CTA-pair kernel from K = 2048 up (7168 -> 2048: 469 vs 512 us)
// and loses at K = 896 and at T <= 8192, where its per-tile epilogue and
// pipeline fill dominate.
static bool sparse_preferred(int64_t T, int64_t K, int64_t O, int num_sms) {
    (void)O;
    (void)num_sms;
    return T >= 16384 && K >= 2048;
}

// The forward behind sbl_linear_path and sbl_linear_rmsnorm: with g the
// activations are RMS-normalised by the front-end kernel before quantisation,
// and the decode sizes take the warp-MMA kernel on the quantised activations.
// check_only: run every host-side argument check and return before anything
// is enqueued.
static sbl_status linear_impl(const uint16_t* x_bf16, const float* g, float eps, int64_t T, int64_t K,
                              const uint8_t* packed, const float* row_scale, int64_t O, int n, int m, void* y,
                              int y_dtype, int32_t* acc_out, void* workspace, size_t workspace_bytes, int path,
                              void* stream, bool check_only = false) {
    if (T < 0 || O < 0) return SBL_ERR_INVALID_ARG;
    if (sbl_status s = check_k(K)) return s;
    if (g) {
        if (!(eps >= 0.0f) || !(eps < 3.0e38f)) return SBL_ERR_INVALID_ARG;
        if (T > 0 && O > 0 && !aligned(g, 16)) return SBL_ERR_INVALID_ARG;
    }
    if (!nm_ok(n, m)) return SBL_ERR_UNSUPPORTED;
    if (y_dtype != SBL_F32 && y_dtype != SBL_BF16) return SBL_ERR_INVALID_ARG;
    if (path < SBL_PATH_AUTO || path > SBL_PATH_PREFILL_SPARSE) return SBL_ERR_INVALID_ARG;
    if (path == SBL_PATH_PREFILL_SPARSE && !sparse_eligible(K, n, m)) return SBL_ERR_UNSUPPORTED;
    const bool forced_prefill = path >= SBL_PATH_PREFILL;
    if (forced_prefill && K % 64 != 0) return SBL_ERR_UNSUPPORTED;
    if (T == 0 || O == 0) return SBL_OK;
    if (!x_bf16 || !packed || !row_scale || !y) return SBL_ERR_INVALID_ARG;
    if (!aligned(x_bf16, 16) || !aligned(packed, 16) || !aligned(row_scale, 16) || !aligned(y, 16))
        return SBL_ERR_INVALID_ARG;
    if (acc_out && !aligned(acc_out, 16)) return SBL_ERR_INVALID_ARG;
    if (T > (1ll << 31) - 1 || O > (1ll << 31) - 1) return SBL_ERR_UNSUPPORTED;
    const size_t need = base_workspace_bytes(T, K);
    if (!workspace || workspace_bytes < need || !aligned(workspace, 256)) return SBL_ERR_WORKSPACE;
    // the sparse path runs only in a workspace that also holds the compressed weights
    const size_t sparse_need = sparse_eligible(K, n, m) ? need + sbl::sp_scratch_bytes(O, K) : 0;
    const bool sparse_fits = sparse_need != 0 && workspace_bytes >= sparse_need;
    if (path == SBL_PATH_PREFILL_SPARSE && !sparse_fits) return SBL_ERR_WORKSPACE;
    bool prefill = forced_prefill;
    if (path == SBL_PATH_AUTO) prefill = ((T > kDecodeMaxTokens) || (K > kDecodeMaxK)) && (K % 64 == 0);
    if (!prefill && K > kDecodeMaxK) return SBL_ERR_UNSUPPORTED;
    if (g && !prefill && !sbl::decode_mma_supported(K)) return SBL_ERR_UNSUPPORTED;
    if (check_only) return SBL_OK;

    DeviceInfo* d;
    if (sbl_status s = device_info(&d)) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int8_t* xq = static_cast<int8_t*>(workspace);
    float* s_tok = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + round256(static_cast<size_t>(T) * K));
    // the activation front end: absmax quantisation, RMSNorm first when g is given
    auto front = [&](int layout, void* zero16, long long nzero16) {
        return g ? sbl::launch_rmsnorm_quant(x_bf16, g, eps, T, K, xq, s_tok, layout, d->status, st, zero16, nzero16)
                 : sbl::launch_quant(x_bf16, T, K, xq, s_tok, layout, d->status, st, zero16, nzero16);
    };

    const int ybf = y_dtype == SBL_BF16 ? 1 : 0;
    cudaError_t e;
    const bool sparse = prefill && sparse_fits && (path == SBL_PATH_PREFILL_SPARSE ||
                                                   (path <= SBL_PATH_PREFILL && sparse_preferred(T, K, O, d->num_sms)));
    if (sparse) {
        uint8_t* scratch = static_cast<uint8_t*>(workspace) + need;
        e = front(sbl::kLayoutNatural, nullptr, 0);
        if (e != cudaSuccess) return SBL_ERR_CUDA;
        e = sbl::launch_prefill_sp(xq, s_tok, T, K, packed, row_scale, O, y, ybf, acc_out, scratch, d->status,
                                   d->num_sms, st);
    } else if (prefill) {
        // a split along k when the one-CTA tiles would leave most SMs idle and
        // the workspace holds the accumulator tiles, which the quantisation
        // kernel zeroes
        int ksplit = 1;
        int32_t* part = nullptr;
        long long nzero16 = 0;
        if (path != SBL_PATH_PREFILL_PAIR) {
            int ks = 1;
            const size_t sb = split_bytes(T, K, O, d->num_sms, &ks);
            if (ks > 1 && workspace_bytes >= need + sb) {
                ksplit = ks;
                part = reinterpret_cast<int32_t*>(static_cast<uint8_t*>(workspace) + need);
                nzero16 = static_cast<long long>(sb / 16);
            }
        }
        e = front(sbl::kLayoutPairs, part, nzero16);
        if (e != cudaSuccess) return SBL_ERR_CUDA;
        const int variant = path == SBL_PATH_PREFILL_1CTA ? sbl::kPrefillOneCta
                            : path == SBL_PATH_PREFILL_PAIR ? sbl::kPrefillPair
                                                            : sbl::kPrefillAuto;
        e = sbl::launch_prefill(xq, s_tok, T, K, packed, row_scale, O, y, ybf, acc_out, d->status, d->num_sms, variant,
                                ksplit, part, st);
    } else if (g) {
        // RMSNorm front end, then the warp-MMA decode on the quantised activations
        e = front(sbl::kLayoutPairs, nullptr, 0);
        if (e != cudaSuccess) return SBL_ERR_CUDA;
        e = sbl::launch_decode_mma(packed, row_scale, O, K, x_bf16, T, y, ybf, acc_out, d->status, d->num_sms, st, xq,
                                   s_tok);
    } else {
        // the decode kernels quantise the activations themselves
        if (T >= kDecodeMmaMinTokens && sbl::decode_mma_supported(K))
            e = sbl::launch_decode_mma(packed, row_scale, O, K, x_bf16, T, y, ybf, acc_out, d->status, d->num_sms, st);
        else
            e = sbl::launch_decode(packed, row_scale, O, K, x_bf16, T, y, ybf, acc_out, d->status, d->num_sms, st);
    }
    return from_cuda(e);
}

sbl_status sbl_linear_path(const uint16_t* x_bf16, int64_t T, int64_t K, const uint8_t* packed,
                           const float* row_scale, int64_t O, int n, int m, void* y, int y_dtype, int32_t* acc_out,
                           void* workspace, size_t workspace_bytes, int path, void* stream) {
    return linear_impl(x_bf16, nullptr, 0.0f, T, K, packed, row_scale, O, n, m, y, y_dtype, acc_out, workspace,
                       workspace_bytes, path, stream);
}

sbl_status sbl_linear_rmsnorm(const uint16_t* x_bf16, const float* g, float eps, int64_t T, int64_t K,
                              const uint8_t* packed, const float* row_scale, int64_t O, int n, int m, void* y,
                              int y_dtype, int32_t* acc_out, void* workspace, size_t workspace_bytes, int path,
                              void* stream) {
    if (!g) return SBL_ERR_INVALID_ARG;
    return linear_impl(x_bf16, g, eps, T, K, packed, row_scale, O, n, m, y, y_dtype, acc_out, workspace,
                       workspace_bytes, path, stream);
}

// The contraction on activations the caller quantised already (x_q in column
// order and s_tok, as sbl_quant_act writes them).  The sparse GEMM reads that
// order as it is; the dense GEMMs and the warp-MMA decode read the pairing
// order, which xq_to_pairs_kernel writes into the workspace.
sbl_status sbl_linear_q(const int8_t* x_q, const float* s_tok, int64_t T, int64_t K, const uint8_t* packed,
                        const float* row_scale, int64_t O, int n, int m, void* y, int y_dtype, int32_t* acc_out,
                        void* workspace, size_t workspace_bytes, void* stream) {
    if (T < 0 || O < 0) return SBL_ERR_INVALID_ARG;
    if (sbl_status s = check_k(K)) return s;
    if (!nm_ok(n, m)) return SBL_ERR_UNSUPPORTED;
    if (y_dtype != SBL_F32 && y_dtype != SBL_BF16) return SBL_ERR_INVALID_ARG;
    if (K % 64 != 0) return SBL_ERR_UNSUPPORTED;
    if (T == 0 || O == 0) return SBL_OK;
    if (!x_q || !s_tok || !packed || !row_scale || !y) return SBL_ERR_INVALID_ARG;
    if (!aligned(x_q, 16) || !aligned(s_tok, 16) || !aligned(packed, 16) || !aligned(row_scale, 16) ||
        !aligned(y, 16))
        return SBL_ERR_INVALID_ARG;
    if (acc_out && !aligned(acc_out, 16)) return SBL_ERR_INVALID_ARG;
    if (T > (1ll << 31) - 1 || O > (1ll << 31) - 1) return SBL_ERR_UNSUPPORTED;
    const bool prefill = T > kDecodeMaxTokens || K > kDecodeMaxK;
    if (!prefill && !sbl::decode_mma_supported(K)) return SBL_ERR_UNSUPPORTED;
    const size_t need = base_workspace_bytes(T, K);
    if (!workspace || workspace_bytes < need || !aligned(workspace, 256)) return SBL_ERR_WORKSPACE;

    DeviceInfo* d;
    if (sbl_status s = device_info(&d)) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int ybf = y_dtype == SBL_BF16 ? 1 : 0;
    const size_t sparse_need = sparse_eligible(K, n, m) ? need + sbl::sp_scratch_bytes(O, K) : 0;
    if (prefill && sparse_need != 0 && workspace_bytes >= sparse_need && sparse_preferred(T, K, O, d->num_sms))
        return from_cuda(sbl::launch_prefill_sp(x_q, s_tok, T, K, packed, row_scale, O, y, ybf, acc_out,
                                                static_cast<uint8_t*>(workspace) + need, d->status, d->num_sms, st));
    int8_t* xp = static_cast<int8_t*>(workspace);
    cudaError_t e = sbl::launch_xq_to_pairs(x_q, T, K, xp, d->num_sms, st);
    if (e != cudaSuccess) return SBL_ERR_CUDA;
    if (prefill)
        e = sbl::launch_prefill(xp, s_tok, T, K, packed, row_scale, O, y, ybf, acc_out, d->status, d->num_sms,
                                sbl::kPrefillAuto, 1, nullptr, st);
    else
        e = sbl::launch_decode_mma(packed, row_scale, O, K, nullptr, T, y, ybf, acc_out, d->status, d->num_sms, st, xp,
                                   s_tok);
    return from_cuda(e);
}

sbl_status sbl_copy_to_device(void* device_dst, const void* host_src, size_t bytes, void* stream) {
    if (bytes == 0) return SBL_OK;
    if (!device_dst || !host_src) return SBL_ERR_INVALID_ARG;
    return from_cuda(cudaMemcpyAsync(device_dst, host_src, bytes, cudaMemcpyHostToDevice,
                                     static_cast<cudaStream_t>(stream)));
}

sbl_status sbl_copy_to_host(void* host_dst, const void* device_src, size_t bytes, void* stream) {
    if (bytes == 0) return SBL_OK;
    if (!host_dst || !device_src) return SBL_ERR_INVALID_ARG;
    return from_cuda(cudaMemcpyAsync(host_dst, device_src, bytes, cudaMemcpyDeviceToHost,
                                     static_cast<cudaStream_t>(stream)));
}

sbl_status sbl_linear_hostio(const uint16_t* x_host, int64_t T, int64_t K, uint16_t* x_dev, const uint8_t* packed,
                             const float* row_scale, int64_t O, int n, int m, void* y_dev, void* y_host, int y_dtype,
                             void* workspace, size_t workspace_bytes, void* stream) {
    // every check first, so that an argument error enqueues nothing
    if (sbl_status s = linear_impl(x_dev, nullptr, 0.0f, T, K, packed, row_scale, O, n, m, y_dev, y_dtype, nullptr,
                                   workspace, workspace_bytes, SBL_PATH_AUTO, stream, true))
        return s;
    if (T == 0 || O == 0) return SBL_OK;
    if (!x_host || !y_host) return SBL_ERR_INVALID_ARG;
    const size_t x_bytes = static_cast<size_t>(T) * static_cast<size_t>(K) * 2;
    const size_t y_bytes = static_cast<size_t>(T) * static_cast<size_t>(O) * (y_dtype == SBL_BF16 ? 2 : 4);
    if (sbl_status s = sbl_copy_to_device(x_dev, x_host, x_bytes, stream)) return s;
    if (sbl_status s = linear_impl(x_dev, nullptr, 0.0f, T, K, packed, row_scale, O, n, m, y_dev, y_dtype, nullptr,
                                   workspace, workspace_bytes, SBL_PATH_AUTO, stream))
        return s;
    return sbl_copy_to_host(y_host, y_dev, y_bytes, stream);
}

sbl_status sbl_linear(const uint16_t* x_bf16, int64_t T, int64_t K, const uint8_t* packed, const float* row_scale,
                      int64_t O, int n, int m, void* y, int y_dtype, int32_t* acc_out, void* workspace,
                      size_t workspace_bytes, void* stream) {
    return sbl_linear_path(x_bf16, T, K, packed, row_scale, O, n, m, y, y_dtype, acc_out, workspace,
                           workspace_bytes, SBL_PATH_AUTO, stream);
}

size_t sbl_linear_grouped_workspace_bytes(int64_t T, int64_t K) {
    if (T <= 0 || K <= 0) return 0;
    return base_workspace_bytes(T, K);
}

sbl_status sbl_linear_grouped(const uint16_t* x_bf16, int64_t T, int64_t K, int G, const uint8_t* const* packed,
                              const float* const* row_scale, const int64_t* O, int n, int m, void* const* y,
                              int y_dtype, int32_t* const* acc_out, void* workspace, size_t workspace_bytes,
                              void* stream) {
    if (G < 1 || G > SBL_MAX_GROUP || G > sbl::decode_max_group() || !packed || !row_scale || !O || !y)
        return SBL_ERR_INVALID_ARG;
    if (T < 0) return SBL_ERR_INVALID_ARG;
    if (sbl_status s = check_k(K)) return s;
    if (!nm_ok(n, m)) return SBL_ERR_UNSUPPORTED;
    if (y_dtype != SBL_F32 && y_dtype != SBL_BF16) return SBL_ERR_INVALID_ARG;
    long long rows = 0;
    for (int g = 0; g < G; ++g) {
        if (O[g] < 0 || O[g] > (1ll << 31) - 1) return SBL_ERR_INVALID_ARG;
        rows += O[g];
        if (T > 0 && O[g] > 0) {
            if (!packed[g] || !row_scale[g] || !y[g]) return SBL_ERR_INVALID_ARG;
            if (!aligned(packed[g], 16) || !aligned(row_scale[g], 16) || !aligned(y[g], 16)) return SBL_ERR_INVALID_ARG;
            if (acc_out && acc_out[g] && !aligned(acc_out[g], 16)) return SBL_ERR_INVALID_ARG;
        }
    }
    if (T == 0 || rows == 0) return SBL_OK;
    if (!x_bf16 || !aligned(x_bf16, 16)) return SBL_ERR_INVALID_ARG;
    if (T > (1ll << 31) - 1) return SBL_ERR_UNSUPPORTED;
    const bool prefill = ((T > kDecodeMaxTokens) || (K > kDecodeMaxK)) && (K % 64 == 0);
    if (!prefill && K > kDecodeMaxK) return SBL_ERR_UNSUPPORTED;
    const size_t need = base_workspace_bytes(T, K);
    if (prefill && (!workspace || workspace_bytes < need || !aligned(workspace, 256))) return SBL_ERR_WORKSPACE;
    DeviceInfo* d;
    if (sbl_status s = device_info(&d)) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int ybf = y_dtype == SBL_BF16 ? 1 : 0;
    cudaError_t e = cudaSuccess;
    if (!prefill && !(T >= kDecodeMmaMinTokens && sbl::decode_mma_supported(K))) {
        // one launch streams every matrix's weights; the kernel quantises x once per block
        long long Ol[SBL_MAX_GROUP];
        for (int g = 0; g < G; ++g) Ol[g] = O[g];
        e = sbl::launch_decode_grouped(G, packed, row_scale, Ol, K, x_bf16, T, y, ybf, acc_out, d->status,
                                       d->num_sms, st);
    } else if (!prefill) {
        // warp-level MMA decode, one launch per matrix
        for (int g = 0; g < G && e == cudaSuccess; ++g)
            if (O[g] > 0)
                e = sbl::launch_decode_mma(packed[g], row_scale[g], O[g], K, x_bf16, T, y[g], ybf,
                                           acc_out ? acc_out[g] : nullptr, d->status, d->num_sms, st);
    } else {
        // x quantised once (pairing order), then the dense tensor-core GEMM per matrix
        int8_t* xq = static_cast<int8_t*>(workspace);
        float* s_tok = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + round256(static_cast<size_t>(T) * K));
        e = sbl::launch_quant(x_bf16, T, K, xq, s_tok, sbl::kLayoutPairs, d->status, st);
        // the non-empty layers, up to prefill_max_group() per launch of the one-CTA kernel
        const uint8_t* gp[SBL_MAX_GROUP];
        const float* gs[SBL_MAX_GROUP];
        long long go[SBL_MAX_GROUP];
        void* gy[SBL_MAX_GROUP];
        int32_t* ga[SBL_MAX_GROUP];
        int n_l = 0;
        for (int g = 0; g < G; ++g)
            if (O[g] > 0) {
                gp[n_l] = packed[g];
                gs[n_l] = row_scale[g];
                go[n_l] = O[g];
                gy[n_l] = y[g];
                ga[n_l] = acc_out ? acc_out[g] : nullptr;
                ++n_l;
            }
        const int per = sbl::prefill_max_group();
        for (int g0 = 0; g0 < n_l && e == cudaSuccess; g0 += per) {
            const int cnt = n_l - g0 < per ? n_l - g0 : per;
            e = sbl::launch_prefill_grouped(xq, s_tok, T, K, cnt, gp + g0, gs + g0, go + g0, gy + g0, ybf, ga + g0,
                                            d->status, d->num_sms, st);
        }
    }
    return from_cuda(e);
}

int64_t sbl_decode_max_tokens(void) { return kDecodeMaxTokens; }

int sbl_linear_plan(int64_t T, int64_t K, int64_t O, int n, int m, size_t workspace_bytes) {
    if (T <= 0 || O <= 0) return -static_cast<int>(SBL_ERR_INVALID_ARG);
    if (sbl_status s = check_k(K)) return -static_cast<int>(s);
    if (!nm_ok(n, m)) return -static_cast<int>(SBL_ERR_UNSUPPORTED);
    const bool prefill = ((T > kDecodeMaxTokens) || (K > kDecodeMaxK)) && (K % 64 == 0);
    if (!prefill) return K > kDecodeMaxK ? -static_cast<int>(SBL_ERR_UNSUPPORTED) : SBL_PATH_DECODE;
    const size_t need = base_workspace_bytes(T, K);
    if (workspace_bytes < need) return -static_cast<int>(SBL_ERR_WORKSPACE);
    DeviceInfo* d;
    if (sbl_status s = device_info(&d)) return -static_cast<int>(s);
    if (sparse_eligible(K, n, m) && workspace_bytes >= need + sbl::sp_scratch_bytes(O, K) &&
        sparse_preferred(T, K, O, d->num_sms))
        return SBL_PATH_PREFILL_SPARSE;
    int ks = 1;
    const size_t sb = split_bytes(T, K, O, d->num_sms, &ks);
    if (ks > 1 && workspace_bytes >= need + sb) return SBL_PATH_PREFILL_1CTA;
    return sbl::choose_dense_prefill(T, O, d->num_sms, nullptr) == 2 ? SBL_PATH_PREFILL_PAIR : SBL_PATH_PREFILL_1CTA;
}

sbl_status sbl_device_status(void* stream) {
    DeviceInfo* d;
    if (sbl_status s = device_info(&d)) return s;
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return SBL_ERR_CUDA;
    unsigned word = 0;
    if (cudaMemcpy(&word, d->status, sizeof(word), cudaMemcpyDeviceToHost) != cudaSuccess) return SBL_ERR_CUDA;
    const unsigned zero = 0;
    if (cudaMemcpy(d->status, &zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess) return SBL_ERR_CUDA;
    if (word & sbl::kStatusTimeout) return SBL_ERR_TIMEOUT;
    if (word & sbl::kStatusNonfinite) return SBL_ERR_NONFINITE;
    if (word & sbl::kStatusInvalid) return SBL_ERR_INVALID_ARG;
    return SBL_OK;
}

sbl_status sbl_selftest_bounded_wait(uint32_t max_polls, void* stream) {
    DeviceInfo* d;
    if (sbl_status s = device_info(&d)) return s;
    sbl::bounded_wait_selftest<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(max_polls, d->status);
    if (cudaGetLastError() != cudaSuccess) return SBL_ERR_CUDA;
    return sbl_device_status(stream);
}

const char* sbl_status_string(sbl_status s) {
    switch (s) {
        case SBL_OK: return "ok";
        case SBL_ERR_INVALID_ARG: return "invalid argument";
        case SBL_ERR_UNSUPPORTED: return "unsupported pattern or shape";
        case SBL_ERR_NONFINITE: return "non-finite input seen on the device";
        case SBL_ERR_CUDA: return "CUDA error";
        case SBL_ERR_TIMEOUT: return "bounded device wait ran out";
        case SBL_ERR_WORKSPACE: return "workspace missing, too small or unaligned";
    }
    return "unknown status";
}

const char* sbl_version(void) { return "sbl 0.1.0 (sm_100a)"; }

#ifdef SBL_TRACE
// Debug builds only: device buffer of 16 x 256 uint64 for prefill event stamps, shared by the
// one-CTA and the CTA-pair kernels (NULL disables).
sbl_status sbl_debug_set_trace(void* buf) {
    const cudaError_t e = sbl::set_prefill_trace(buf);
    return from_cuda(e != cudaSuccess ? e : sbl::set_pair_trace(buf));
}
#endif

}  // extern "C"
