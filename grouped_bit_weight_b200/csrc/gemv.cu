// gemv.cu -- bandwidth-targeted grouped GEMV for decode-sized batches.
//
// "grouped-nf4-gemm 0.43.0", release notes at the top of the page: on GPUs
// with many SMs, single-request decode at Qwen3-30B-A3B's expert shapes uses
// a bandwidth-targeted GEMV instead of the tensor-core GEMM.  With one
// routed row per expert every weight byte is used once, so the kernel is
// bound by HBM: it streams each packed row with 16-byte loads straight into
// registers and never touches the tensor cores.
//
// Decode: a 256-entry pair table in shared memory maps one packed byte to
// the fp32 values of its two codes (exact codebook values), so one 64-bit
// shared load decodes two weights.  Each lane owns its own 8-byte column of
// the table (entry b of lane l at b*256 + l*8), which makes every lookup
// bank-conflict free, and the entry address is built from the byte with one
// byte-permute.  The block scale multiplies the per-chunk partial sum
// (sum_k C[q_k] x_k) * scale, and fp32x2 FMAs accumulate.
//
// Work: output element (p, n) is one task = one weight row against one
// routed row.  Tasks are split into contiguous ranges, one per group of G
// lanes; a lane owns CPL 16-byte chunks (32 weights each) of the row.  Loads
// for the next D tasks are kept in flight while the current one is reduced.
#include "common.cuh"

namespace gbw {
namespace {

__constant__ float kNF4g[16] = {
    -1.0f,
    -0.6961928009986877f,
    -0.5250730514526367f,
    -0.39491748809814453f,
    -0.28444138169288635f,
    -0.18477343022823334f,
    -0.09105003625154495f,
    0.0f,
    0.07958029955625534f,
    0.16093020141124725f,
    0.24611230194568634f,
    0.33791524171829224f,
    0.44070982933044434f,
    0.5626170039176941f,
    0.7229568362236023f,
    1.0f,
};
__constant__ float kE2M1g[8] = {0.0f, 0.5f, 1.0f, 1.5f, 2.0f, 3.0f, 4.0f, 6.0f};

constexpr int kThreads = 384;  // 12 warps: up to 170 registers a thread
constexpr int kLutBytes = 256 * 256;  // 256 entries x 32 lanes x 8 bytes

__device__ __forceinline__ float code_value(Fmt F, uint32_t q) {
  if (F == Fmt::NF4) return kNF4g[q];
  const float m = kE2M1g[q & 7u];
  return (q & 8u) ? -m : m;
}

__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}

__device__ __forceinline__ uint64_t pack2(float lo, float hi) {
  return (uint64_t)__float_as_uint(lo) | ((uint64_t)__float_as_uint(hi) << 32);
}

__device__ __forceinline__ float sum2(uint64_t v) {
  return __uint_as_float((uint32_t)v) + __uint_as_float((uint32_t)(v >> 32));
}

__device__ __forceinline__ uint64_t lds64(uint32_t addr) {
  uint64_t v;
  asm volatile("ld.shared.b64 %0, [%1];" : "=l"(v) : "r"(addr));
  return v;
}

// Scale of chunk c (32 weights) of a row.
template <Fmt F>
__device__ __forceinline__ float chunk_scale(const void* scale, int64_t row,
                                             int64_t K, int64_t c) {
  if (F == Fmt::NF4)
    return __ldg(reinterpret_cast<const float*>(scale) + row * (K / 64) + (c >> 1));
  const uint32_t s = __ldg(reinterpret_cast<const uint8_t*>(scale) + row * (K / 32) + c);
  if (s == 0xFFu) return __int_as_float(0x7FC00000);
  if (s == 0u) return __int_as_float(0x00400000);
  return __int_as_float((int)(s << 23));
}

template <Fmt F, int G, int CPL, int D>
__global__ void __launch_bounds__(kThreads, 1)
gemv_kernel(GroupedProblem pb) {
  extern __shared__ __align__(1024) uint8_t smem[];
  int32_t* off_s = reinterpret_cast<int32_t*>(smem + kLutBytes);

  // pair table: entry b -> (value of even element, value of odd element)
  for (int i = threadIdx.x; i < 256 * 32; i += kThreads) {
    const uint32_t b = (uint32_t)i >> 5, l = (uint32_t)i & 31u;
    const uint32_t qe = (F == Fmt::NF4) ? (b >> 4) : (b & 15u);
    const uint32_t qo = (F == Fmt::NF4) ? (b & 15u) : (b >> 4);
    *reinterpret_cast<uint64_t*>(smem + b * 256 + l * 8) =
        pack2(code_value(F, qe), code_value(F, qo));
  }
  load_offsets_clamped(pb.offsets, pb.E, pb.P, off_s, pb.err);

  const int64_t K = pb.K, N = pb.N;
  const int64_t C = K / 32;                       // 16-byte chunks per row
  const int64_t per_pass = (int64_t)G * CPL;
  const int npass = (int)((C + per_pass - 1) / per_pass);
  const int lane = threadIdx.x & 31;
  const int li = lane % G;                        // lane within its group
  const uint32_t lut = smem_u32(smem);
  const uint32_t lanebits = (uint32_t)lane << 3;  // this lane's table column

  const int64_t groups_per_block = (kThreads / 32) * (32 / G);
  const int64_t gid = blockIdx.x * groups_per_block + (threadIdx.x >> 5) * (32 / G) + lane / G;
  const int64_t ngroups = (int64_t)gridDim.x * groups_per_block;
  const int64_t total = pb.P * N;
  const int64_t begin = total * gid / ngroups;
  const int64_t end = total * (gid + 1) / ngroups;

  // x of the current routed row, fp32 pairs; valid for (xp, pass 0).
  uint64_t xr[CPL][16];
  int64_t xp = -1;

  uint4 pk[D][CPL];
  float sc[D][CPL];

  auto row_of = [&](int64_t t, int64_t& p, int64_t& n) {
    p = t / N;
    n = t - p * N;
    const int32_t e = expert_of_row(off_s, pb.E, (int32_t)p);
    return (int64_t)e * N + n;  // weight row
  };
  auto issue = [&](int d, int64_t t, int pass) {
    int64_t p, n;
    const int64_t wrow = row_of(t, p, n);
    const uint4* src = reinterpret_cast<const uint4*>(pb.w + wrow * (K / 2));
#pragma unroll
    for (int i = 0; i < CPL; ++i) {
      const int64_t c = pass * per_pass + (int64_t)i * G + li;
      if (c < C) {
        pk[d][i] = __ldg(src + c);
        sc[d][i] = chunk_scale<F>(pb.scale, wrow, K, c);
      } else {
        pk[d][i] = make_uint4(0x77777777u, 0x77777777u, 0x77777777u, 0x77777777u);
        sc[d][i] = 0.0f;
      }
    }
  };
  auto load_x = [&](int64_t p, int pass) {
    const int32_t tok = token_of_row(pb.row_to_token, (int32_t)p, pb.T, pb.err);
    const uint4* xs = reinterpret_cast<const uint4*>(pb.x + (int64_t)tok * K);
#pragma unroll
    for (int i = 0; i < CPL; ++i) {
      const int64_t c = pass * per_pass + (int64_t)i * G + li;
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        uint4 q = make_uint4(0, 0, 0, 0);
        if (c < C) q = __ldg(xs + c * 4 + v);
        const uint32_t w4[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
        for (int j = 0; j < 4; ++j)
          xr[i][v * 4 + j] = pack2(__uint_as_float(w4[j] << 16),
                                   __uint_as_float(w4[j] & 0xFFFF0000u));
      }
    }
  };
  auto dot = [&](const uint4 (&q)[CPL], const float (&s)[CPL]) {
    float acc = 0.0f;
#pragma unroll
    for (int i = 0; i < CPL; ++i) {
      const uint32_t w4[4] = {q[i].x, q[i].y, q[i].z, q[i].w};
      uint64_t a2 = 0;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
#pragma unroll
        for (int b = 0; b < 4; ++b) {
          const uint32_t addr = lut + prmt(w4[j], lanebits, 0x5504u | (b << 4));
          a2 = fma2(lds64(addr), xr[i][j * 4 + b], a2);
        }
      }
      acc = fmaf(sum2(a2), s[i], acc);
    }
    return acc;
  };

  // Whole warps run the loop the same number of times (shuffles inside).
  const int64_t my_n = end - begin;
  int64_t max_n = my_n;
#pragma unroll
  for (int o = G; o < 32; o <<= 1)
    max_n = max(max_n, __shfl_xor_sync(0xffffffffu, max_n, o));

  if (npass == 1) {
#pragma unroll
    for (int d = 0; d < D; ++d)
      if (d < my_n) issue(d, begin + d, 0);
    for (int64_t i0 = 0; i0 < max_n; i0 += D) {
#pragma unroll
      for (int d = 0; d < D; ++d) {
        const int64_t i = i0 + d;
        const bool live = i < my_n;
        float acc = 0.0f;
        if (live) {
          const int64_t t = begin + i;
          const int64_t p = t / N;
          if (p != xp) { load_x(p, 0); xp = p; }
          acc = dot(pk[d], sc[d]);
          if (i + D < my_n) issue(d, t + D, 0);
        }
        if (i < max_n) {
#pragma unroll
          for (int o = G / 2; o; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o, G);
          if (live && li == 0)
            pb.out[begin + i] = __bfloat16_as_ushort(__float2bfloat16_rn(acc));
        }
      }
    }
  } else {
    // Rows longer than one pass: x is reloaded per pass, no prefetch.
    for (int64_t i = 0; i < max_n; ++i) {
      const bool live = i < my_n;
      float acc = 0.0f;
      if (live) {
        const int64_t t = begin + i;
        const int64_t p = t / N;
        for (int pass = 0; pass < npass; ++pass) {
          load_x(p, pass);
          issue(0, t, pass);
          acc += dot(pk[0], sc[0]);
        }
      }
#pragma unroll
      for (int o = G / 2; o; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o, G);
      if (live && li == 0)
        pb.out[begin + i] = __bfloat16_as_ushort(__float2bfloat16_rn(acc));
    }
  }
}

template <Fmt F, int G, int CPL>
cudaError_t launch_gc(const GroupedProblem& pb, int num_sms, cudaStream_t s) {
  constexpr int D = CPL == 1 ? 8 : (CPL == 2 ? 4 : (CPL == 3 ? 2 : 1));
  const size_t smem = kLutBytes + sizeof(int32_t) * (size_t)(pb.E + 1);
  auto k = gemv_kernel<F, G, CPL, D>;
  cudaError_t e = cudaFuncSetAttribute(
      k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  k<<<num_sms, kThreads, smem, s>>>(pb);
  return cudaGetLastError();
}

template <Fmt F>
cudaError_t launch_f(const GroupedProblem& pb, int num_sms, cudaStream_t s) {
  const int64_t C = pb.K / 32;
  // pick lanes-per-row G and chunks-per-lane CPL with the fewest idle slots
  int bestG = 32, bestCPL = 4;
  int64_t best_idle = INT64_MAX;
  for (int G : {32, 16, 8}) {
    int64_t cpl = (C + G - 1) / G;
    int64_t npass = 1;
    if (cpl > 4) { npass = (C + 4 * G - 1) / (4 * G); cpl = 4; }
    const int64_t idle = npass * cpl * G - C;
    if (idle < best_idle) { best_idle = idle; bestG = G; bestCPL = (int)cpl; }
  }
#define GBW_GEMV_CASE(GG, CC) \
  if (bestG == GG && bestCPL == CC) return launch_gc<F, GG, CC>(pb, num_sms, s);
  GBW_GEMV_CASE(32, 1) GBW_GEMV_CASE(32, 2) GBW_GEMV_CASE(32, 3) GBW_GEMV_CASE(32, 4)
  GBW_GEMV_CASE(16, 1) GBW_GEMV_CASE(16, 2) GBW_GEMV_CASE(16, 3) GBW_GEMV_CASE(16, 4)
  GBW_GEMV_CASE(8, 1) GBW_GEMV_CASE(8, 2) GBW_GEMV_CASE(8, 3) GBW_GEMV_CASE(8, 4)
#undef GBW_GEMV_CASE
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_gemv(Fmt f, const GroupedProblem& pb, int num_sms,
                        cudaStream_t s) {
  if (pb.P == 0 || pb.N == 0) return cudaSuccess;
  return f == Fmt::NF4 ? launch_f<Fmt::NF4>(pb, num_sms, s)
                       : launch_f<Fmt::MXFP4>(pb, num_sms, s);
}

}  // namespace gbw
