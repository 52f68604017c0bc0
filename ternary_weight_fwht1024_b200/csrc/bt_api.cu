// C ABI of libbt.so: host-side validation and dispatch (declared in include/bt.h).
#include <atomic>

#include "bt_internal.cuh"

namespace bt {
cudaError_t launch_pack(int layout, const int8_t* trits, int64_t N, int64_t K, uint8_t* codes,
                        int32_t* dev_err, cudaStream_t stream);
cudaError_t launch_unpack(int layout, const uint8_t* codes, int64_t N, int64_t K, int8_t* trits,
                          int32_t* dev_err, cudaStream_t stream);
cudaError_t launch_fwht1024(const uint16_t* x, const int8_t* sign, int64_t M, int64_t K,
                            int out_dtype, void* out, int num_sms, cudaStream_t stream);
size_t gemv_workspace_bytes(int layout, int64_t M, int64_t N, int64_t K, int num_sms);
cudaError_t launch_gemv(int layout, const uint8_t* codes, const uint16_t* scales, const void* x,
                        int x_dtype, const int8_t* sign, int64_t M, int64_t N, int64_t K, int y_dtype,
                        void* y, void* workspace, int32_t* dev_err, int num_sms, cudaStream_t stream);
size_t gemv_noalloc_max_bytes();
cudaError_t gemv_noalloc_scratch(void** out);
size_t gemv1_workspace_bytes(int layout, const DecodeProblem* problems, int count);
bool gemv_lut_applies(int layout, int64_t M, int64_t K, const void* codes, const void* scales);
cudaError_t launch_gemv_lut(int layout, const uint8_t* codes, const uint16_t* scales, const void* x, int x_bf16,
                            const int8_t* sign, int M, int64_t N, int64_t K, int y_dtype, void* y, void* workspace,
                            int32_t* dev_err, int num_sms, cudaStream_t stream);
cudaError_t launch_gemv1(int layout, const DecodeProblem* problems, int count, const int8_t* sign, int y_dtype,
                         void* workspace, int32_t* dev_err, int num_sms, cudaStream_t stream);
size_t gemm_workspace_bytes(int layout, int64_t M, int64_t N, int64_t K, int num_sms);
size_t ternarize_workspace_bytes(int64_t N, int64_t K);
cudaError_t launch_ternarize(const float* W, const int8_t* sign, int64_t N, int64_t K, int8_t* trits,
                             uint16_t* scales, void* workspace, cudaStream_t stream);
cudaError_t launch_gemm(int layout, const uint8_t* codes, const uint16_t* scales, const void* x,
                        int x_dtype, const int8_t* sign, int64_t M, int64_t N, int64_t K, void* y,
                        void* workspace, int32_t* dev_err, int num_sms, cudaStream_t stream);
}  // namespace bt

namespace {

constexpr int kVersion = 1;
constexpr int kDefaultSms = 148;   // B200; used when no device can be queried

// SM count of the current device, looked up once per device ordinal. Without
// a usable device (a build or test machine) every query would retry the
// driver's initialisation, so a failed query is remembered too.
int current_sm_count() {
    static std::atomic<int> no_device{0};
    static std::atomic<int> cached[64];
    if (no_device.load(std::memory_order_relaxed)) return kDefaultSms;
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        no_device.store(1, std::memory_order_relaxed);
        return kDefaultSms;
    }
    if (dev >= 0 && dev < 64) {
        const int c = cached[dev].load(std::memory_order_relaxed);
        if (c > 0) return c;
    }
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0) {
        cudaGetLastError();
        return kDefaultSms;
    }
    if (dev >= 0 && dev < 64) cached[dev].store(sms, std::memory_order_relaxed);
    return sms;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }
bool valid_layout(int layout) { return layout == BT_LAYOUT_B3 || layout == BT_LAYOUT_2BIT || layout == BT_LAYOUT_B3C; }
bool valid_dtype(int d) { return d == BT_F32 || d == BT_BF16; }
int64_t group_bytes(int layout) { return layout == BT_LAYOUT_B3 ? 26 : 32; }

// A failed launch also leaves its error as the runtime's last error; clear it,
// so that a later call does not report it as its own.
bt_status from_cuda(cudaError_t e) {
    if (e == cudaSuccess) return BT_OK;
    cudaGetLastError();
    return BT_ERR_CUDA;
}

// Shared validation of the product entry points.
bt_status check_product_args(int layout, const uint8_t* codes, const uint16_t* scales, const void* x,
                             int x_dtype, const int8_t* sign, int64_t M, int64_t N, int64_t K,
                             const void* y) {
    if (!valid_layout(layout) || !valid_dtype(x_dtype)) return BT_ERR_INVALID_ARG;
    if (M < 0 || N < 0 || K < 0) return BT_ERR_SHAPE;
    if (K % 128 != 0) return BT_ERR_SHAPE;
    if (sign && (K % 1024 != 0 || x_dtype != BT_BF16)) return sign && x_dtype != BT_BF16 ? BT_ERR_INVALID_ARG : BT_ERR_SHAPE;
    if (K > (int64_t(1) << 30) || N > (int64_t(1) << 30)) return BT_ERR_SHAPE;
    if (M == 0 || N == 0) return BT_OK;
    if (!y) return BT_ERR_INVALID_ARG;
    if (K > 0 && (!codes || !scales || !x)) return BT_ERR_INVALID_ARG;
    if (!aligned(codes, 16) || !aligned(scales, 4) || !aligned(x, 16) || !aligned(y, 16) || !aligned(sign, 16))
        return BT_ERR_ALIGN;
    return BT_OK;
}

// y = 0 for K = 0 (the empty sum)
__global__ void zero_kernel(uint8_t* p, int64_t bytes) {
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < bytes; i += (int64_t)gridDim.x * blockDim.x)
        p[i] = 0;
}

cudaError_t launch_zero(void* p, int64_t bytes, cudaStream_t s) {
    if (bytes <= 0) return cudaSuccess;
    int blocks = static_cast<int>((bytes + 255) / 256);
    if (blocks > 1024) blocks = 1024;
    zero_kernel<<<blocks, 256, 0, s>>>(static_cast<uint8_t*>(p), bytes);
    return cudaGetLastError();
}

}  // namespace

extern "C" {

const char* bt_status_string(int status) {
    switch (status) {
        case BT_OK: return "ok";
        case BT_ERR_INVALID_ARG: return "invalid argument (NULL pointer or bad enum)";
        case BT_ERR_SHAPE: return "shape constraint violated";
        case BT_ERR_ALIGN: return "pointer misaligned";
        case BT_ERR_WORKSPACE: return "workspace missing or too small";
        case BT_ERR_UNSUPPORTED: return "unsupported request";
        case BT_ERR_CUDA: return "CUDA launch or query failed";
        default: return "unknown status";
    }
}

int bt_version(void) { return kVersion; }

int64_t bt_codes_row_bytes(int layout, int64_t K) {
    if (!valid_layout(layout) || K <= 0 || K % 128 != 0) return -1;
    if (layout == BT_LAYOUT_B3C) return ((K + 4) / 5 + 15) / 16 * 16;
    return (K / 128) * group_bytes(layout);
}

bt_status bt_pack(int layout, const int8_t* trits, int64_t N, int64_t K, uint8_t* codes,
                  int32_t* dev_err, void* stream) {
    if (!valid_layout(layout)) return BT_ERR_INVALID_ARG;
    if (N < 0 || K < 0 || K % 128 != 0) return BT_ERR_SHAPE;
    if (N == 0 || K == 0) return BT_OK;
    if (!trits || !codes) return BT_ERR_INVALID_ARG;
    if (!aligned(trits, 4) || !aligned(dev_err, 4)) return BT_ERR_ALIGN;
    return from_cuda(bt::launch_pack(layout, trits, N, K, codes, dev_err, static_cast<cudaStream_t>(stream)));
}

bt_status bt_unpack(int layout, const uint8_t* codes, int64_t N, int64_t K, int8_t* trits,
                    int32_t* dev_err, void* stream) {
    if (!valid_layout(layout)) return BT_ERR_INVALID_ARG;
    if (N < 0 || K < 0 || K % 128 != 0) return BT_ERR_SHAPE;
    if (N == 0 || K == 0) return BT_OK;
    if (!trits || !codes) return BT_ERR_INVALID_ARG;
    if (!aligned(trits, 4) || !aligned(dev_err, 4)) return BT_ERR_ALIGN;
    return from_cuda(bt::launch_unpack(layout, codes, N, K, trits, dev_err, static_cast<cudaStream_t>(stream)));
}

bt_status bt_fwht1024(const uint16_t* x_bf16, const int8_t* sign1024, int64_t M, int64_t K,
                      int out_dtype, void* x_rot, void* stream) {
    if (!valid_dtype(out_dtype)) return BT_ERR_INVALID_ARG;
    if (M < 0 || K < 0 || K % 1024 != 0) return BT_ERR_SHAPE;
    if (M == 0 || K == 0) return BT_OK;
    if (!x_bf16 || !sign1024 || !x_rot) return BT_ERR_INVALID_ARG;
    if (!aligned(x_bf16, 16) || !aligned(sign1024, 16) || !aligned(x_rot, 16)) return BT_ERR_ALIGN;
    return from_cuda(bt::launch_fwht1024(x_bf16, sign1024, M, K, out_dtype, x_rot, current_sm_count(),
                                         static_cast<cudaStream_t>(stream)));
}

// The continuous base-3 layout runs on the single-row table-lookup kernel
// only: M = 1, K % 1024 == 0, codes and scales on 16-byte boundaries.
bt_status check_b3c(int layout, int64_t M, int64_t K, const void* codes, const void* scales) {
    if (layout != BT_LAYOUT_B3C) return BT_OK;
    if (M > 1 || K % 1024 != 0) return BT_ERR_SHAPE;
    if (!aligned(codes, 16) || !aligned(scales, 16)) return BT_ERR_ALIGN;
    return BT_OK;
}

size_t bt_gemv_workspace_bytes(int layout, int64_t M, int64_t N, int64_t K) {
    if (!valid_layout(layout) || M < 1 || M > 16 || N < 1 || K < 128 || K % 128 != 0) return 0;
    if (layout == BT_LAYOUT_B3C && (M > 1 || K % 1024 != 0)) return 0;
    return bt::gemv_workspace_bytes(layout, M, N, K, current_sm_count());
}

// One GEMV call on a validated workspace: products whose weights TMA can
// stream take the persistent kernels of bt_gemv_lut.cu (table lookup for
// M = 1, tensor cores above), the rest the kernels of bt_gemv.cu.
cudaError_t run_gemv(int layout, const uint8_t* codes, const uint16_t* scales, const void* x, int x_dtype,
                     const int8_t* sign1024, int64_t M, int64_t N, int64_t K, int y_dtype, void* y, void* ws,
                     int32_t* dev_err, int sms, cudaStream_t s) {
    // Base-3 weights at 2 <= M <= 8 stay on the TMA-fed kernel of bt_gemv.cu,
    // which was measured faster there (27B-equivalent sweep at M = 4); above
    // M = 8, and for the 2-bit layout, the tensor-core kernel of
    // bt_gemv_lut.cu streams the weights once for all rows.
    const bool old_path = layout == BT_LAYOUT_B3 && M >= 2 && M <= 8;
    if (!old_path && bt::gemv_lut_applies(layout, M, K, codes, scales))
        return bt::launch_gemv_lut(layout, codes, scales, x, x_dtype == BT_BF16 ? 1 : 0, sign1024, (int)M, N, K,
                                   y_dtype, y, ws, dev_err, sms, s);
    return bt::launch_gemv(layout, codes, scales, x, x_dtype, sign1024, M, N, K, y_dtype, y, ws, dev_err, sms, s);
}

bt_status bt_gemv(int layout, const uint8_t* codes, const uint16_t* scales, const void* x, int x_dtype,
                  const int8_t* sign1024, int64_t M, int64_t N, int64_t K, int y_dtype, void* y,
                  void* workspace, size_t workspace_bytes, int32_t* dev_err, void* stream) {
    bt_status st = check_product_args(layout, codes, scales, x, x_dtype, sign1024, M, N, K, y);
    if (st != BT_OK) return st;
    if (!valid_dtype(y_dtype)) return BT_ERR_INVALID_ARG;
    if (M > 16) return BT_ERR_SHAPE;
    if ((st = check_b3c(layout, M, K, codes, scales)) != BT_OK) return st;
    if (M == 0 || N == 0) return BT_OK;
    if (!aligned(dev_err, 4)) return BT_ERR_ALIGN;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (K == 0) return from_cuda(launch_zero(y, M * N * (y_dtype == BT_BF16 ? 2 : 4), s));
    const int sms = current_sm_count();
    const size_t need = bt::gemv_workspace_bytes(layout, M, N, K, sms);
    if (!workspace || workspace_bytes < need) return BT_ERR_WORKSPACE;
    if (!aligned(workspace, 256)) return BT_ERR_ALIGN;
    return from_cuda(run_gemv(layout, codes, scales, x, x_dtype, sign1024, M, N, K, y_dtype, y, workspace,
                              dev_err, sms, s));
}

size_t bt_gemv_batched_workspace_bytes(int layout, const bt_gemv_problem* problems, int count) {
    if (!valid_layout(layout) || !problems || count < 1 || count > 256) return 0;
    bt::DecodeProblem dp[256];
    for (int i = 0; i < count; ++i) {
        const bt_gemv_problem& q = problems[i];
        if (q.N < 1 || q.K < 1024 || q.K % 1024 != 0) return 0;
        dp[i] = bt::DecodeProblem{nullptr, nullptr, nullptr, 1, q.x_from, nullptr, q.N, q.K};
    }
    return bt::gemv1_workspace_bytes(layout, dp, count);
}

bt_status bt_gemv_batched(int layout, const bt_gemv_problem* problems, int count, const int8_t* sign1024,
                          int y_dtype, void* workspace, size_t workspace_bytes, int32_t* dev_err, void* stream) {
    if (!valid_layout(layout) || !valid_dtype(y_dtype)) return BT_ERR_INVALID_ARG;
    if (count < 0 || count > 256) return BT_ERR_SHAPE;
    if (count == 0) return BT_OK;
    if (!problems) return BT_ERR_INVALID_ARG;
    if (!aligned(dev_err, 4) || !aligned(sign1024, 16)) return BT_ERR_ALIGN;
    bt::DecodeProblem dp[256];
    for (int i = 0; i < count; ++i) {
        const bt_gemv_problem& q = problems[i];
        if (q.N < 1 || q.K < 1024 || q.K % 1024 != 0 || q.K > (int64_t(1) << 30) || q.N > (int64_t(1) << 24))
            return BT_ERR_SHAPE;
        if (!q.codes || !q.scales || !q.y) return BT_ERR_INVALID_ARG;
        if (!aligned(q.codes, 16) || !aligned(q.scales, 16) || !aligned(q.y, 16)) return BT_ERR_ALIGN;
        if (q.x_from >= 0) {
            if (q.x_from >= i) return BT_ERR_INVALID_ARG;             // only earlier outputs
            if (problems[q.x_from].N != q.K) return BT_ERR_SHAPE;     // that output is this input
            if (sign1024 && y_dtype != BT_BF16) return BT_ERR_INVALID_ARG;  // rotation reads bf16
        } else {
            if (q.x_from != -1) return BT_ERR_INVALID_ARG;
            if (!q.x || !valid_dtype(q.x_dtype)) return BT_ERR_INVALID_ARG;
            if (sign1024 && q.x_dtype != BT_BF16) return BT_ERR_INVALID_ARG;
            if (!aligned(q.x, 16)) return BT_ERR_ALIGN;
        }
        dp[i] = bt::DecodeProblem{q.codes, q.scales, q.x, q.x_from >= 0 ? (y_dtype == BT_BF16 ? 1 : 0)
                                                                        : (q.x_dtype == BT_BF16 ? 1 : 0),
                                  q.x_from, q.y, q.N, q.K};
    }
    const size_t need = bt_gemv_batched_workspace_bytes(layout, problems, count);
    if (!workspace || workspace_bytes < need) return BT_ERR_WORKSPACE;
    if (!aligned(workspace, 256)) return BT_ERR_ALIGN;
    return from_cuda(bt::launch_gemv1(layout, dp, count, sign1024, y_dtype, workspace, dev_err, current_sm_count(),
                                      static_cast<cudaStream_t>(stream)));
}

bt_status bt_gemv_noalloc(int layout, const uint8_t* codes, const uint16_t* scales, const void* x,
                          int x_dtype, const int8_t* sign1024, int64_t M, int64_t N, int64_t K, int y_dtype,
                          void* y, int32_t* dev_err, void* stream) {
    bt_status st = check_product_args(layout, codes, scales, x, x_dtype, sign1024, M, N, K, y);
    if (st != BT_OK) return st;
    if (!valid_dtype(y_dtype)) return BT_ERR_INVALID_ARG;
    if (M > 16) return BT_ERR_SHAPE;
    if ((st = check_b3c(layout, M, K, codes, scales)) != BT_OK) return st;
    if (M == 0 || N == 0) return BT_OK;
    if (!aligned(dev_err, 4)) return BT_ERR_ALIGN;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (K == 0) return from_cuda(launch_zero(y, M * N * (y_dtype == BT_BF16 ? 2 : 4), s));
    const int sms = current_sm_count();
    if (bt::gemv_workspace_bytes(layout, M, N, K, sms) > bt::gemv_noalloc_max_bytes()) return BT_ERR_WORKSPACE;
    void* scratch = nullptr;
    if (bt::gemv_noalloc_scratch(&scratch) != cudaSuccess) { cudaGetLastError(); return BT_ERR_CUDA; }
    return from_cuda(run_gemv(layout, codes, scales, x, x_dtype, sign1024, M, N, K, y_dtype, y, scratch, dev_err,
                              sms, s));
}

size_t bt_gemm_workspace_bytes(int layout, int64_t M, int64_t N, int64_t K) {
    if (!valid_layout(layout) || layout == BT_LAYOUT_B3C || M < 128 || M % 128 != 0 || N < 128 || N % 128 != 0 || K < 128 || K % 128 != 0)
        return 0;
    return bt::gemm_workspace_bytes(layout, M, N, K, current_sm_count());
}

bt_status bt_gemm(int layout, const uint8_t* codes, const uint16_t* scales, const void* x, int x_dtype,
                  const int8_t* sign1024, int64_t M, int64_t N, int64_t K, void* y_bf16,
                  void* workspace, size_t workspace_bytes, int32_t* dev_err, void* stream) {
    bt_status st = check_product_args(layout, codes, scales, x, x_dtype, sign1024, M, N, K, y_bf16);
    if (st != BT_OK) return st;
    if (layout == BT_LAYOUT_B3C) return BT_ERR_INVALID_ARG;  // the prefill GEMM reads group-aligned bytes
    if (M == 0 || N == 0) return BT_OK;
    if (M % 128 != 0 || N % 128 != 0) return BT_ERR_SHAPE;
    if (!aligned(dev_err, 4)) return BT_ERR_ALIGN;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (K == 0) return from_cuda(launch_zero(y_bf16, M * N * 2, s));
    const int sms = current_sm_count();
    const size_t need = bt::gemm_workspace_bytes(layout, M, N, K, sms);
    if (!workspace || workspace_bytes < need) return BT_ERR_WORKSPACE;
    if (!aligned(workspace, 256)) return BT_ERR_ALIGN;
    return from_cuda(bt::launch_gemm(layout, codes, scales, x, x_dtype, sign1024, M, N, K, y_bf16,
                                     workspace, dev_err, sms, s));
}

size_t bt_ternarize_workspace_bytes(int64_t N, int64_t K) {
    if (N < 0 || K < 0 || K % 1024 != 0) return 0;
    return bt::ternarize_workspace_bytes(N, K);
}

bt_status bt_ternarize(const float* W, const int8_t* sign1024, int64_t N, int64_t K, int8_t* trits,
                       uint16_t* scales, void* workspace, size_t workspace_bytes, void* stream) {
    if (N < 0 || K < 0 || K % 1024 != 0 || K > (int64_t(1) << 30) || N > (int64_t(1) << 30)) return BT_ERR_SHAPE;
    if (N == 0 || K == 0) return BT_OK;
    if (!W || !sign1024 || !trits || !scales) return BT_ERR_INVALID_ARG;
    if (!aligned(W, 16) || !aligned(sign1024, 16) || !aligned(scales, 2)) return BT_ERR_ALIGN;
    if (!workspace || workspace_bytes < bt::ternarize_workspace_bytes(N, K)) return BT_ERR_WORKSPACE;
    if (!aligned(workspace, 256)) return BT_ERR_ALIGN;
    return from_cuda(bt::launch_ternarize(W, sign1024, N, K, trits, scales, workspace,
                                          static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
