// api.cu -- the extern "C" entry points declared in include/gbw.h: host-side
// argument checks, the sm_100 check, the per-device error word and the
// choice between the tensor-core GEMM and the bandwidth GEMV.
#include <stdio.h>
#include <string.h>

#include <mutex>

#include "common.cuh"

namespace gbw {
namespace {

// GBW_DEVERR_* bits raised by the kernels of this library on this device,
// and the copy of it that gbw_device_status takes atomically.
__device__ int g_err_word;
__device__ int g_err_copy;

constexpr int kMaxDevices = 64;
// Experts per call: the kernels keep expert_offsets in shared memory.
constexpr int32_t kMaxExperts = 1024;

// Per-device state, set up once per device (std::call_once, so host threads
// that make their first calls at the same time see it complete).
struct DeviceState {
  int* err = nullptr;   // device address of g_err_word
  int* copy = nullptr;  // device address of g_err_copy
  int sms = 0;
  int arch_ok = 0;      // 1 sm_100, -1 other
  cudaError_t init = cudaSuccess;
};
DeviceState g_dev[kMaxDevices];
std::once_flag g_dev_once[kMaxDevices];

thread_local char g_msg[256] = "";

gbw_status launch_error(cudaError_t e) {
  snprintf(g_msg, sizeof(g_msg), "CUDA error: %s", cudaGetErrorString(e));
  return GBW_ERR_LAUNCH;
}

// Architecture check, SM count and the device addresses of the error word
// and its copy (resolved with the device current).
gbw_status device_state(int** err, int* sms, int** copy = nullptr) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return launch_error(e);
  if (dev < 0 || dev >= kMaxDevices) return GBW_ERR_ARCH;
  DeviceState& d = g_dev[dev];
  std::call_once(g_dev_once[dev], [&]() {
    int major = 0, minor = 0, n = 0;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (major != 10 || minor != 0) {
      d.arch_ok = -1;
      return;
    }
    void* p = nullptr;
    void* c = nullptr;
    d.init = cudaGetSymbolAddress(&p, g_err_word);
    if (d.init == cudaSuccess) d.init = cudaGetSymbolAddress(&c, g_err_copy);
    if (d.init != cudaSuccess) return;
    d.err = static_cast<int*>(p);
    d.copy = static_cast<int*>(c);
    d.sms = n;
    d.arch_ok = 1;
  });
  if (d.init != cudaSuccess) return launch_error(d.init);
  if (d.arch_ok < 0) {
    snprintf(g_msg, sizeof(g_msg), "device %d is not sm_100 (B200)", dev);
    return GBW_ERR_ARCH;
  }
  *err = d.err;
  *sms = d.sms;
  if (copy) *copy = d.copy;
  return GBW_OK;
}

// Takes the error word in one atomic step (and clears it when asked), so a
// bit a kernel on another stream raises at the same time is either in the
// copy or still in the word, never lost.
__global__ void take_error_word(int* err, int* copy, int clear) {
  *copy = clear ? atomicExch(err, 0) : atomicOr(err, 0);
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

gbw_status fail(gbw_status s, const char* what) {
  snprintf(g_msg, sizeof(g_msg), "%s", what);
  return s;
}

gbw_status grouped_forward(Fmt f, const uint16_t* x, int64_t T, int64_t K,
                           const uint8_t* w, const void* scale, int32_t E,
                           int64_t N, const int32_t* offsets,
                           const int32_t* row_to_token, int64_t P,
                           uint16_t* out, int32_t mode, void* stream) {
  if (T < 0 || K <= 0 || N <= 0 || E < 1 || P < 0)
    return fail(GBW_ERR_SHAPE, "need T >= 0, K > 0, N > 0, E >= 1, P >= 0");
  if (f == Fmt::NF4 && K % 64) return fail(GBW_ERR_SHAPE, "NF4 needs K % 64 == 0");
  if (f == Fmt::MXFP4 && K % 32) return fail(GBW_ERR_SHAPE, "MXFP4 needs K % 32 == 0");
  if (N % 8) return fail(GBW_ERR_SHAPE, "N must be a multiple of 8");
  if (K > (int64_t)1 << 30 || N > (int64_t)1 << 30 || P > INT32_MAX ||
      T > INT32_MAX || (int64_t)E * N > INT32_MAX)
    return fail(GBW_ERR_SHAPE, "sizes exceed the 32-bit row indices");
  const int32_t flags = mode & ~0xFF;
  mode &= 0xFF;
  if (mode < GBW_MODE_AUTO || mode > GBW_MODE_GEMV || (flags & ~GBW_FLAG_OVERLAP_PREV))
    return fail(GBW_ERR_SHAPE, "unknown mode or flag");
  if (E > kMaxExperts) return fail(GBW_ERR_SHAPE, "at most 1024 experts");
  if (!offsets || !w || !scale) return fail(GBW_ERR_NULL, "NULL weights or offsets");
  if (P > 0 && (!x || !out)) return fail(GBW_ERR_NULL, "NULL x or out");
  if (!row_to_token && T < P)
    return fail(GBW_ERR_SHAPE, "row_to_token == NULL needs T >= P");
  if (row_to_token && P > 0 && T < 1) return fail(GBW_ERR_SHAPE, "T must be >= 1");
  if (!aligned16(x) || !aligned16(w) || !aligned16(out))
    return fail(GBW_ERR_ALIGN, "x, packed weights and out must be 16-byte aligned");
  if (f == Fmt::NF4 && !aligned4(scale)) return fail(GBW_ERR_ALIGN, "absmax must be 4-byte aligned");
  if (f == Fmt::MXFP4 && (reinterpret_cast<uintptr_t>(scale) & 1u))
    return fail(GBW_ERR_ALIGN, "MXFP4 scales must be 2-byte aligned");
  if (!aligned4(offsets) || (row_to_token && !aligned4(row_to_token)))
    return fail(GBW_ERR_ALIGN, "offsets / row_to_token must be 4-byte aligned");
  int* err = nullptr;
  int sms = 0;
  gbw_status st = device_state(&err, &sms);
  if (st != GBW_OK) return st;
  if (P == 0) return GBW_OK;
  GroupedProblem pb{x, T, K, w, scale, E, N, offsets, row_to_token, P, out, err, flags};
  const bool fits = gemv_fits(f, pb, sms);
  if (mode == GBW_MODE_GEMV && !fits)
    return fail(GBW_ERR_SHAPE, "rows too long for the GEMV's shared-memory ring");
  // AUTO: the bandwidth GEMV while experts average at most four routed rows
  // (it streams each active expert's weights once and beats the tensor-core
  // GEMM there: measured on B200 at Qwen3-30B-A3B shapes, the GEMM wins from
  // about six rows per expert); the GEMM takes K % 64 == 32 (MXFP4) with a
  // half last stage
  const bool gemv = mode == GBW_MODE_GEMV ||
                    (mode == GBW_MODE_AUTO && fits && P <= 4 * (int64_t)E);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = gemv ? launch_gemv(f, pb, sms, s) : launch_gemm(f, pb, sms, s);
  return e == cudaSuccess ? GBW_OK : launch_error(e);
}

}  // namespace
}  // namespace gbw

using namespace gbw;

extern "C" {

gbw_status gnf4_grouped_gemm(const uint16_t* x, int64_t T, int64_t K,
                             const uint8_t* packed, const float* absmax,
                             int32_t E, int64_t N,
                             const int32_t* expert_offsets,
                             const int32_t* row_to_token, int64_t P,
                             uint16_t* out, int32_t mode, void* stream) {
  return grouped_forward(Fmt::NF4, x, T, K, packed, absmax, E, N,
                         expert_offsets, row_to_token, P, out, mode, stream);
}

gbw_status gmxfp4_grouped_gemm(const uint16_t* x, int64_t T, int64_t K,
                               const uint8_t* blocks, const uint8_t* scales,
                               int32_t E, int64_t N,
                               const int32_t* expert_offsets,
                               const int32_t* row_to_token, int64_t P,
                               uint16_t* out, int32_t mode, void* stream) {
  return grouped_forward(Fmt::MXFP4, x, T, K, blocks, scales, E, N,
                         expert_offsets, row_to_token, P, out, mode, stream);
}

static gbw_status grouped_dgrad(Fmt f, const uint16_t* dy, int64_t P, int64_t N,
                                const uint8_t* packed, const void* scale, int32_t E,
                                int64_t K, const int32_t* expert_offsets, uint16_t* dx,
                                void* stream) {
  if (P < 0 || N <= 0 || K <= 0 || E < 1)
    return fail(GBW_ERR_SHAPE, "need P >= 0, N > 0, K > 0, E >= 1");
  if (K % 64 || N % 64) return fail(GBW_ERR_SHAPE, "dgrad needs K % 64 == 0 and N % 64 == 0");
  if (E > kMaxExperts) return fail(GBW_ERR_SHAPE, "at most 1024 experts");
  if (K > (int64_t)1 << 30 || P > INT32_MAX || (int64_t)E * N > INT32_MAX)
    return fail(GBW_ERR_SHAPE, "sizes exceed the 32-bit row indices");
  if (!packed || !scale || !expert_offsets) return fail(GBW_ERR_NULL, "NULL weights or offsets");
  if (P > 0 && (!dy || !dx)) return fail(GBW_ERR_NULL, "NULL dy or dx");
  if (!aligned16(dy) || !aligned16(packed) || !aligned16(dx))
    return fail(GBW_ERR_ALIGN, "dy, packed and dx must be 16-byte aligned");
  if ((f == Fmt::NF4 ? !aligned4(scale) : (reinterpret_cast<uintptr_t>(scale) & 1u) != 0) ||
      !aligned4(expert_offsets))
    return fail(GBW_ERR_ALIGN, "absmax 4-byte, scales 2-byte, offsets 4-byte aligned");
  int* err = nullptr;
  int sms = 0;
  gbw_status st = device_state(&err, &sms);
  if (st != GBW_OK) return st;
  if (P == 0) return GBW_OK;
  GroupedProblem pb{dy, P, K, packed, scale, E, N, expert_offsets, nullptr, P, dx, err, 0};
  cudaError_t e = launch_dgrad(f, pb, sms, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? GBW_OK : launch_error(e);
}

gbw_status gnf4_grouped_dgrad(const uint16_t* dy, int64_t P, int64_t N,
                              const uint8_t* packed, const float* absmax,
                              int32_t E, int64_t K,
                              const int32_t* expert_offsets, uint16_t* dx,
                              void* stream) {
  return grouped_dgrad(Fmt::NF4, dy, P, N, packed, absmax, E, K, expert_offsets, dx, stream);
}

gbw_status gmxfp4_grouped_dgrad(const uint16_t* dy, int64_t P, int64_t N,
                                const uint8_t* blocks, const uint8_t* scales,
                                int32_t E, int64_t K,
                                const int32_t* expert_offsets, uint16_t* dx,
                                void* stream) {
  return grouped_dgrad(Fmt::MXFP4, dy, P, N, blocks, scales, E, K, expert_offsets, dx, stream);
}

static gbw_status expert_mlp(Fmt f, const uint16_t* x, int64_t T, int64_t H,
                             const uint8_t* gu, const void* gu_scale, const uint8_t* dn,
                             const void* dn_scale, int32_t E, int64_t I,
                             const int32_t* offsets, const int32_t* row_to_token, int64_t P,
                             uint16_t* h, uint16_t* out, int32_t mode, void* stream) {
  if (T < 0 || H <= 0 || I <= 0 || E < 1 || P < 0)
    return fail(GBW_ERR_SHAPE, "need T >= 0, H > 0, I > 0, E >= 1, P >= 0");
  if (H % 64 || I % 64)
    return fail(GBW_ERR_SHAPE, "the fused expert pass needs H % 64 == 0 and I % 64 == 0");
  if (H > (int64_t)1 << 30 || I > (int64_t)1 << 29 || P > INT32_MAX || T > INT32_MAX ||
      (int64_t)E * 2 * I > INT32_MAX || (int64_t)E * H > INT32_MAX)
    return fail(GBW_ERR_SHAPE, "sizes exceed the 32-bit row indices");
  if (mode < GBW_MODE_AUTO || mode > GBW_MODE_GEMV)
    return fail(GBW_ERR_SHAPE, "unknown mode (the fused pass takes no flags)");
  if (E > kMaxExperts) return fail(GBW_ERR_SHAPE, "at most 1024 experts");
  if (!offsets || !gu || !gu_scale || !dn || !dn_scale)
    return fail(GBW_ERR_NULL, "NULL weights or offsets");
  if (P > 0 && (!x || !h || !out)) return fail(GBW_ERR_NULL, "NULL x, h or out");
  if (!row_to_token && T < P) return fail(GBW_ERR_SHAPE, "row_to_token == NULL needs T >= P");
  if (row_to_token && P > 0 && T < 1) return fail(GBW_ERR_SHAPE, "T must be >= 1");
  if (!aligned16(x) || !aligned16(gu) || !aligned16(dn) || !aligned16(h) || !aligned16(out))
    return fail(GBW_ERR_ALIGN, "x, packed weights, h and out must be 16-byte aligned");
  if (f == Fmt::NF4 && (!aligned4(gu_scale) || !aligned4(dn_scale)))
    return fail(GBW_ERR_ALIGN, "absmax must be 4-byte aligned");
  if (f == Fmt::MXFP4 && ((reinterpret_cast<uintptr_t>(gu_scale) | reinterpret_cast<uintptr_t>(dn_scale)) & 1u))
    return fail(GBW_ERR_ALIGN, "MXFP4 scales must be 2-byte aligned");
  if (!aligned4(offsets) || (row_to_token && !aligned4(row_to_token)))
    return fail(GBW_ERR_ALIGN, "offsets / row_to_token must be 4-byte aligned");
  int* err = nullptr;
  int sms = 0;
  gbw_status st = device_state(&err, &sms);
  if (st != GBW_OK) return st;
  if (P == 0) return GBW_OK;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // gate_up with SwiGLU fused into the output (h = silu(gate) * up), then
  // down over h (row p of h is routed row p); both on the bandwidth GEMV or
  // both on the tensor cores
  const bool gemv = mode == GBW_MODE_GEMV || (mode == GBW_MODE_AUTO && P <= 4 * (int64_t)E);
  GroupedProblem g{x, T, H, gu, gu_scale, E, 2 * I, offsets, row_to_token, P, h, err, 0};
  cudaError_t e = gemv ? launch_gemv(f, g, sms, s, true) : launch_gemm(f, g, sms, s, I);
  if (e != cudaSuccess) return launch_error(e);
  GroupedProblem d{h, P, I, dn, dn_scale, E, H, offsets, nullptr, P, out, err, 0};
  e = gemv ? launch_gemv(f, d, sms, s) : launch_gemm(f, d, sms, s);
  return e == cudaSuccess ? GBW_OK : launch_error(e);
}

gbw_status gnf4_grouped_expert_mlp(const uint16_t* x, int64_t T, int64_t H,
                                   const uint8_t* gu_packed, const float* gu_absmax,
                                   const uint8_t* dn_packed, const float* dn_absmax,
                                   int32_t E, int64_t I, const int32_t* expert_offsets,
                                   const int32_t* row_to_token, int64_t P, uint16_t* h,
                                   uint16_t* out, int32_t mode, void* stream) {
  return expert_mlp(Fmt::NF4, x, T, H, gu_packed, gu_absmax, dn_packed, dn_absmax, E, I,
                    expert_offsets, row_to_token, P, h, out, mode, stream);
}

gbw_status gmxfp4_grouped_expert_mlp(const uint16_t* x, int64_t T, int64_t H,
                                     const uint8_t* gu_blocks, const uint8_t* gu_scales,
                                     const uint8_t* dn_blocks, const uint8_t* dn_scales,
                                     int32_t E, int64_t I, const int32_t* expert_offsets,
                                     const int32_t* row_to_token, int64_t P, uint16_t* h,
                                     uint16_t* out, int32_t mode, void* stream) {
  return expert_mlp(Fmt::MXFP4, x, T, H, gu_blocks, gu_scales, dn_blocks, dn_scales, E, I,
                    expert_offsets, row_to_token, P, h, out, mode, stream);
}

// ---------------------------------------------------------------------------
// Fused expert pass without any device allocation.
//
// gnf4_grouped_expert_mlp asks the caller for the h workspace.  Some callers
// cannot provide one: a plugin inside an inference engine whose device memory
// is already handed out by the engine, or a serving loop that forbids device
// allocation after warm-up because cudaMalloc can synchronise the device and
// fragments memory a caching allocator holds.  For them the h rows live in a
// fixed array in this library's device image.  Every device that loads the
// library holds the array until the process exits, so it is kept small.
// ---------------------------------------------------------------------------

// h scratch of gnf4_grouped_expert_mlp_noalloc: P * I bf16 values at most.
constexpr int64_t kNoAllocHElems = (int64_t)1 << 21;  // 2,097,152 values, 4 MiB
static __device__ __align__(256) uint16_t g_noalloc_h[kNoAllocHElems];

// Device address of g_noalloc_h per device.  In host code the name
// g_noalloc_h is only a host-side stand-in, so the address is looked up once
// per device, with that device current, on the first call there.
static uint16_t* g_noalloc_ptr[kMaxDevices];
static cudaError_t g_noalloc_err[kMaxDevices];
static std::once_flag g_noalloc_once[kMaxDevices];

gbw_status gnf4_grouped_expert_mlp_noalloc(const uint16_t* x, int64_t T, int64_t H,
                                           const uint8_t* gu_packed, const float* gu_absmax,
                                           const uint8_t* dn_packed, const float* dn_absmax,
                                           int32_t E, int64_t I, const int32_t* expert_offsets,
                                           const int32_t* row_to_token, int64_t P,
                                           uint16_t* out, int32_t mode, void* stream) {
  if (P > 0 && I > 0 && P <= INT32_MAX && I <= ((int64_t)1 << 29) && P * I > kNoAllocHElems) {
    snprintf(g_msg, sizeof(g_msg),
             "P * I = %lld exceeds the %lld bf16 values of the no-allocation h scratch",
             (long long)(P * I), (long long)kNoAllocHElems);
    return GBW_ERR_SHAPE;
  }
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return launch_error(e);
  if (dev < 0 || dev >= kMaxDevices) return GBW_ERR_ARCH;
  std::call_once(g_noalloc_once[dev], [dev]() {
    void* p = nullptr;
    g_noalloc_err[dev] = cudaGetSymbolAddress(&p, g_noalloc_h);
    g_noalloc_ptr[dev] = static_cast<uint16_t*>(p);
  });
  if (g_noalloc_err[dev] != cudaSuccess) return launch_error(g_noalloc_err[dev]);
  // every h element the down projection reads is written by gate_up in the
  // same call, so the array's previous contents never matter
  return expert_mlp(Fmt::NF4, x, T, H, gu_packed, gu_absmax, dn_packed, dn_absmax, E, I,
                    expert_offsets, row_to_token, P, g_noalloc_ptr[dev], out, mode, stream);
}

gbw_status gnf4_dequant(const uint8_t* packed, const float* absmax,
                        int64_t rows, int64_t K, uint16_t* w_out,
                        void* stream) {
  if (rows < 0 || K <= 0 || K % 64) return fail(GBW_ERR_SHAPE, "need rows >= 0, K % 64 == 0");
  if (rows > 0 && (!packed || !absmax || !w_out)) return fail(GBW_ERR_NULL, "NULL argument");
  if (!aligned16(packed) || !aligned16(w_out) || !aligned4(absmax))
    return fail(GBW_ERR_ALIGN, "packed / w_out must be 16-byte aligned");
  int* err = nullptr;
  int sms = 0;
  gbw_status st = device_state(&err, &sms);
  if (st != GBW_OK) return st;
  cudaError_t e = launch_dequant(Fmt::NF4, packed, absmax, rows, K, w_out,
                                 static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? GBW_OK : launch_error(e);
}

gbw_status gmxfp4_dequant(const uint8_t* blocks, const uint8_t* scales,
                          int64_t rows, int64_t K, uint16_t* w_out,
                          void* stream) {
  if (rows < 0 || K <= 0 || K % 32) return fail(GBW_ERR_SHAPE, "need rows >= 0, K % 32 == 0");
  if (rows > 0 && (!blocks || !scales || !w_out)) return fail(GBW_ERR_NULL, "NULL argument");
  if (!aligned16(blocks) || !aligned16(w_out))
    return fail(GBW_ERR_ALIGN, "blocks / w_out must be 16-byte aligned");
  int* err = nullptr;
  int sms = 0;
  gbw_status st = device_state(&err, &sms);
  if (st != GBW_OK) return st;
  cudaError_t e = launch_dequant(Fmt::MXFP4, blocks, scales, rows, K, w_out,
                                 static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? GBW_OK : launch_error(e);
}

gbw_status gnf4_quantize(const float* w, int64_t rows, int64_t K,
                         uint8_t* packed, float* absmax, void* stream) {
  if (rows < 0 || K <= 0 || K % 64) return fail(GBW_ERR_SHAPE, "need rows >= 0, K % 64 == 0");
  if (rows > 0 && (!w || !packed || !absmax)) return fail(GBW_ERR_NULL, "NULL argument");
  if (!aligned16(w) || !aligned4(absmax)) return fail(GBW_ERR_ALIGN, "w must be 16-byte aligned");
  int* err = nullptr;
  int sms = 0;
  gbw_status st = device_state(&err, &sms);
  if (st != GBW_OK) return st;
  cudaError_t e = launch_quantize(Fmt::NF4, w, rows, K, packed, absmax,
                                  static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? GBW_OK : launch_error(e);
}

gbw_status gmxfp4_quantize(const float* w, int64_t rows, int64_t K,
                           uint8_t* blocks, uint8_t* scales, void* stream) {
  if (rows < 0 || K <= 0 || K % 32) return fail(GBW_ERR_SHAPE, "need rows >= 0, K % 32 == 0");
  if (rows > 0 && (!w || !blocks || !scales)) return fail(GBW_ERR_NULL, "NULL argument");
  if (!aligned16(w)) return fail(GBW_ERR_ALIGN, "w must be 16-byte aligned");
  int* err = nullptr;
  int sms = 0;
  gbw_status st = device_state(&err, &sms);
  if (st != GBW_OK) return st;
  cudaError_t e = launch_quantize(Fmt::MXFP4, w, rows, K, blocks, scales,
                                  static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? GBW_OK : launch_error(e);
}

gbw_status gbw_device_status(void* stream, int32_t* host_err, int32_t clear) {
  int* err = nullptr;
  int* copy = nullptr;
  int sms = 0;
  gbw_status st = device_state(&err, &sms, &copy);
  if (st != GBW_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  take_error_word<<<1, 1, 0, s>>>(err, copy, clear ? 1 : 0);
  cudaError_t e = cudaGetLastError();
  int v = 0;
  if (e == cudaSuccess) e = cudaMemcpyAsync(&v, copy, sizeof(int), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return launch_error(e);
  if (host_err) *host_err = v;
  return v ? GBW_ERR_DEVICE : GBW_OK;
}

const char* gbw_status_string(gbw_status s) {
  switch (s) {
    case GBW_OK: return "ok";
    case GBW_ERR_NULL: return g_msg[0] ? g_msg : "NULL pointer";
    case GBW_ERR_SHAPE: return g_msg[0] ? g_msg : "unsupported size";
    case GBW_ERR_ALIGN: return g_msg[0] ? g_msg : "misaligned pointer";
    case GBW_ERR_ARCH: return g_msg[0] ? g_msg : "device is not sm_100";
    case GBW_ERR_LAUNCH: return g_msg[0] ? g_msg : "CUDA launch failed";
    case GBW_ERR_DEVICE: return "device error word set (see GBW_DEVERR_* bits)";
  }
  return "unknown status";
}

int32_t gbw_version(void) { return 100; }

}  // extern "C"
