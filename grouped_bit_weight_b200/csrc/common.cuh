// common.cuh -- device-side building blocks shared by the kernels of
// libgbw: launch arguments, the device error word, bounded mbarrier waits,
// TMA (cp.async.bulk.tensor) and tcgen05 (5th-generation tensor core /
// tensor memory) wrappers for sm_100a.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/gbw.h"

namespace gbw {

// ----------------------------------------------------------------------
// launch arguments
// ----------------------------------------------------------------------

// One grouped projection: routed rows sorted by expert, E experts of weight
// [N, K] in a 4-bit packed format.
struct GroupedProblem {
  const uint16_t* x;       // [T, K] bf16 (forward) or dy [P, N] (dgrad)
  int64_t T;
  int64_t K;
  const uint8_t* w;        // packed codes [E, N, K/2]
  const void* scale;       // NF4: float [E, N, K/64]; MXFP4: uint8 [E, N, K/32]
  int32_t E;
  int64_t N;
  const int32_t* offsets;  // [E+1] device
  const int32_t* row_to_token;  // [P] device or nullptr
  int64_t P;
  uint16_t* out;           // [P, N] bf16 (forward) or dx [P, K] (dgrad)
  int* err;                // device error word
  int32_t flags;           // GBW_FLAG_* bits of the call
};

enum class Fmt : int { NF4 = 0, MXFP4 = 1 };

// Host-side launchers (one per kernel family).  Each returns the CUDA
// error of its launch.
cudaError_t launch_dequant(Fmt f, const uint8_t* w, const void* scale,
                           int64_t rows, int64_t K, uint16_t* out,
                           cudaStream_t s);
cudaError_t launch_quantize(Fmt f, const float* w, int64_t rows, int64_t K,
                            uint8_t* codes, void* scale, cudaStream_t s);
// glu: the SwiGLU gate_up variant (p.N = 2I rows per expert, gate rows then
// up rows); out receives h = silu(gate) * up, [P, I].
cudaError_t launch_gemv(Fmt f, const GroupedProblem& p, int num_sms,
                        cudaStream_t s, bool glu = false);
// Whether the GEMV's shared-memory ring holds two blocks of rows of length K.
bool gemv_fits(Fmt f, const GroupedProblem& p, int num_sms);
// glu_i > 0: the SwiGLU gate_up variant (p.N = 2 * glu_i rows per expert,
// gate rows then up rows); out receives h = silu(gate) * up, [P, glu_i].
cudaError_t launch_gemm(Fmt f, const GroupedProblem& p, int num_sms,
                        cudaStream_t s, int64_t glu_i = 0);
cudaError_t launch_dgrad(Fmt f, const GroupedProblem& p, int num_sms, cudaStream_t s);

// ----------------------------------------------------------------------
// device error word
// ----------------------------------------------------------------------

__device__ __forceinline__ void raise_error(int* err, int bit) {
  if (err) atomicOr(err, bit);
}

// ----------------------------------------------------------------------
// small helpers
// ----------------------------------------------------------------------

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

// Two fp32 -> bf16x2, round to nearest even; `lo` lands in bits 15:0.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t d;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
  return d;
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ----------------------------------------------------------------------
// mbarrier (shared memory barriers with transaction counts)
// ----------------------------------------------------------------------

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(count));
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar,
                                                      uint32_t bytes) {
  asm volatile(
      "mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(
          smem_u32(bar)),
      "r"(bytes)
      : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n"
      " mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Wait budget of every pipeline wait: after this many nanoseconds without
// progress the wait gives up, raises GBW_DEVERR_TIMEOUT and the kernel
// unwinds instead of hanging the GPU.
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s

// Bounded wait for the phase with `parity` to complete.  `abort` is a
// shared flag: once any thread of the CTA has given up, every other wait
// returns false at once.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity,
                                          volatile int* abort, int* err) {
  if (mbar_try_wait(bar, parity)) return true;
  uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 0;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 63u) == 63u) {
      if (*abort) return false;
      if (globaltimer_ns() - t0 > kWaitLimitNs) {
        *abort = 1;
        raise_error(err, GBW_DEVERR_TIMEOUT);
        return false;
      }
    }
  }
}

// Wait that ignores the abort flag, used while unwinding to let copies and
// MMAs already in flight finish before shared or tensor memory is released.
__device__ __forceinline__ void mbar_drain(uint64_t* bar, uint32_t parity) {
  uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 0;; ++it) {
    if (mbar_try_wait(bar, parity)) return;
    if ((it & 63u) == 63u && globaltimer_ns() - t0 > kWaitLimitNs) return;
  }
}

// ----------------------------------------------------------------------
// TMA (tensor memory accelerator)
// ----------------------------------------------------------------------

__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* m) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(m))
               : "memory");
}

// 2-D tiled load of box {c0.., c1..} into shared memory, completion counted
// in bytes on `bar`.
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* m,
                                            int32_t c0, int32_t c1,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_"
      "tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(c0), "r"(c1), "r"(smem_u32(bar))
      : "memory");
}

// Bulk (untiled) asynchronous copy of `bytes` contiguous bytes from global
// to shared memory, completion counted in bytes on `bar`.  Both addresses
// 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_load(void* dst, const void* src,
                                          uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], "
      "[%1], %2, [%3];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// 16-byte asynchronous global -> shared copy (L2 only), grouped with
// commit_group and waited for with wait_group.
__device__ __forceinline__ void cp_async_16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src)
               : "memory");
}
// The same copy with `src_bytes` (0..16) read and the rest of the 16 bytes
// zero-filled; with src_bytes == 0 nothing is read from src.
__device__ __forceinline__ void cp_async_16_fill(uint32_t dst, const void* src,
                                                 uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
               "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait_group() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
// Arrive on `bar` once every cp.async this thread issued so far has landed
// (asynchronously; the barrier's expected count already includes this
// arrival).
__device__ __forceinline__ void cp_async_arrive_noinc(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.wait_all;" ::: "memory");
}
// Orders this thread's view of generic-proxy shared-memory writes before its
// later async-proxy accesses (tensor core operand reads).
__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ----------------------------------------------------------------------
// tcgen05: tensor memory and the 5th-generation MMA
// ----------------------------------------------------------------------

// Allocates `ncols` TMEM columns (power of two >= 32) for this CTA; the
// base address is written to *dst_smem.  Whole warp.
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile(
      "tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
          smem_u32(dst_smem)),
      "r"(ncols)
      : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::
                   : "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile(
      "tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr),
      "r"(ncols)
      : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Arrive on `bar` once every tcgen05 operation this thread issued so far
// has completed.
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 "
      "[%0];" ::"r"(smem_u32(bar))
      : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem]^T, kind::f16 (bf16 inputs, fp32 accum).
__device__ __forceinline__ void tc_mma_ts(uint32_t d_tmem, uint32_t a_tmem,
                                          uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}\n" ::"r"(
          d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T, kind::f16.
__device__ __forceinline__ void tc_mma_ss(uint32_t d_tmem, uint64_t a_desc,
                                          uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(
          d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Instruction descriptor, kind::f16: bf16 A and B, fp32 D, M x N tile.
// a_mn / b_mn select the MN-major (transposed) smem layout.
__host__ __device__ constexpr uint32_t make_idesc_bf16(uint32_t M, uint32_t N,
                                                       uint32_t a_mn,
                                                       uint32_t b_mn) {
  return (1u << 4)            // D format: f32
         | (1u << 7)          // A format: bf16
         | (1u << 10)         // B format: bf16
         | (a_mn << 15)       // A major
         | (b_mn << 16)       // B major
         | ((N >> 3) << 17)   // N / 8
         | ((M >> 4) << 24);  // M / 16
}

// Shared-memory matrix descriptor for a 128-byte-swizzled operand.
//   lbo / sbo: leading / stride byte offsets (see the canonical layouts:
//   K-major -> sbo = distance between 8-row groups; MN-major -> lbo =
//   distance between 64-element atoms along MN, sbo = distance between
//   8-row groups along K).
__device__ __forceinline__ uint64_t make_sdesc_sw128(uint32_t saddr,
                                                     uint32_t lbo,
                                                     uint32_t sbo) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1u << 46;  // descriptor version for sm_100
  d |= (uint64_t)2u << 61;  // layout: SWIZZLE_128B
  return d;
}

// 32 lanes x 32 columns of 32-bit TMEM cells <-> 32 registers per thread:
// thread t of the warp owns lane (warp's lane base + t).
// tcgen05.st reads its source registers and tcgen05.ld writes its
// destination registers asynchronously: the registers belong to the
// operation until tcgen05.wait::st / wait::ld.  The wait therefore sits in
// the same asm statement, so the compiler cannot reuse or read those
// registers in between.
__device__ __forceinline__ void tmem_store_32x32b_x32(uint32_t taddr,
                                                      const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, "
      "%7, %8, %9, %10, %11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, "
      "%22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};\n"
      "tcgen05.wait::st.sync.aligned;" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]),
      "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]),
      "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]),
      "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]),
      "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]),
      "r"(r[30]), "r"(r[31])
      : "memory");
}

__device__ __forceinline__ void tmem_load_32x32b_x32(uint32_t taddr,
                                                     uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, "
      "%8, %9, %10, %11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, "
      "%22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];\n"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
        "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]),
        "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]),
        "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
        "=r"(r[31])
      : "r"(taddr)
      : "memory");
}

// ----------------------------------------------------------------------
// grouped-row bookkeeping
// ----------------------------------------------------------------------

// Loads expert_offsets into shared memory as a clamped running maximum in
// [0, P] (so every row range stays inside the caller's buffers) and flags
// any change the clamp made.  off_s has E+1 entries.  Whole block; valid
// offsets (the normal case) are checked in parallel, only invalid ones take
// the serial clamp.  Split in two so a kernel can issue the loads first and
// do other work while they are in flight.
struct OffsetRegs {
  int32_t v[2], nxt[2];  // offsets[e] and offsets[e + 1], e = tid, tid + blockDim
};

__device__ __forceinline__ OffsetRegs prefetch_offsets(const int32_t* offsets,
                                                       int32_t E) {
  OffsetRegs r;
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const int32_t e = (int32_t)(threadIdx.x + k * blockDim.x);
    r.v[k] = e <= E ? __ldg(offsets + e) : 0;
    r.nxt[k] = e < E ? __ldg(offsets + e + 1) : 0;
  }
  return r;
}

__device__ __forceinline__ void commit_offsets(const OffsetRegs& r,
                                               const int32_t* offsets,
                                               int32_t E, int64_t P,
                                               int32_t* off_s, int* err) {
  int bad = 0;
  auto check = [&](int32_t e, int32_t v, int32_t nxt) {
    off_s[e] = v;
    if (v < 0 || v > (int32_t)P || (e == 0 && v != 0) || (e == E && v != (int32_t)P))
      bad = 1;
    if (e < E && nxt < v) bad = 1;
  };
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const int32_t e = (int32_t)(threadIdx.x + k * blockDim.x);
    if (e <= E) check(e, r.v[k], r.nxt[k]);
  }
  for (int32_t e = (int32_t)(threadIdx.x + 2 * blockDim.x); e <= E; e += blockDim.x)
    check(e, __ldg(offsets + e), e < E ? __ldg(offsets + e + 1) : 0);
  if (__syncthreads_or(bad)) {
    if (threadIdx.x == 0) {
      int32_t prev = 0;
      for (int32_t e = 0; e <= E; ++e) {
        int32_t c = off_s[e] < prev ? prev : off_s[e];
        if (c > (int32_t)P) c = (int32_t)P;
        if (e == 0) c = 0;
        if (e == E) c = (int32_t)P;
        off_s[e] = c;
        prev = c;
      }
      raise_error(err, GBW_DEVERR_OFFSETS);
    }
    __syncthreads();
  }
}

__device__ __forceinline__ void load_offsets_clamped(const int32_t* offsets,
                                                     int32_t E, int64_t P,
                                                     int32_t* off_s, int* err) {
  commit_offsets(prefetch_offsets(offsets, E), offsets, E, P, off_s, err);
}

// Programmatic dependent launch: wait until the kernel launched before this
// one on the stream has completed and its writes are visible (a no-op when
// this kernel was not launched as a dependent); then let the next kernel on
// the stream start its own launch.
__device__ __forceinline__ void grid_dependency_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void grid_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ts[e] = sum over experts e' < e of tiles(e'), ts[E] = total, where
// tiles(e) = per_tile_n * ceil(count(e) / rows_per_tile).  Warp 0 scans 32
// experts at a time with shuffles; the block must sync afterwards.
__device__ __forceinline__ void tile_prefix(const int32_t* off_s, int32_t E,
                                            int32_t rows_per_tile,
                                            int32_t per_tile_n, int32_t* ts) {
  if (threadIdx.x >= 32) return;
  const int lane = threadIdx.x;
  int32_t carry = 0;
  for (int32_t base = 0; base < E; base += 32) {
    const int32_t e = base + lane;
    int32_t v = 0;
    if (e < E) {
      const int32_t cnt = off_s[e + 1] - off_s[e];
      v = per_tile_n * ((cnt + rows_per_tile - 1) / rows_per_tile);
    }
    int32_t incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int32_t t = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += t;
    }
    if (e < E) ts[e] = carry + incl - v;
    carry += __shfl_sync(0xffffffffu, incl, 31);
  }
  if (lane == 0) ts[E] = carry;
}

// Expert whose row range holds row p (binary search, p in [0, P)).
__device__ __forceinline__ int32_t expert_of_row(const int32_t* off_s,
                                                 int32_t E, int32_t p) {
  int32_t lo = 0, hi = E - 1;
  while (lo < hi) {
    int32_t mid = (lo + hi + 1) >> 1;
    if (off_s[mid] <= p) lo = mid; else hi = mid - 1;
  }
  return lo;
}

__device__ __forceinline__ int32_t token_of_row(const int32_t* r2t, int32_t p,
                                                int64_t T, int* err) {
  if (!r2t) return p;
  int32_t t = __ldg(r2t + p);
  if (t < 0 || t >= T) {
    raise_error(err, GBW_DEVERR_TOKEN);
    t = t < 0 ? 0 : (int32_t)(T - 1);
  }
  return t;
}

}  // namespace gbw
