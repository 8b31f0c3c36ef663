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

// Walks output elements (p, n) in order, keeping the expert of row p.
struct TaskCursor {
  int64_t p, n;
  int32_t e;
  __device__ __forceinline__ void start(int64_t t, int64_t N, const int32_t* off,
                                        int32_t E) {
    p = t / N;
    n = t - p * N;
    e = expert_of_row(off, E, (int32_t)p);
  }
  // Moving past the last row leaves e at the last expert (never E or more).
  __device__ __forceinline__ void next(int64_t N, const int32_t* off, int32_t E) {
    if (++n == N) {
      n = 0;
      ++p;
      while (e < E - 1 && off[e + 1] <= p) ++e;
    }
  }
};

template <Fmt F, int G, int CPL, int D>
__global__ void __launch_bounds__(kThreads, 1)
gemv_kernel(GroupedProblem pb) {
  extern __shared__ __align__(1024) uint8_t smem[];
  int32_t* off_s = reinterpret_cast<int32_t*>(smem + kLutBytes);

  const int64_t K = pb.K, N = pb.N;
  const int64_t C = K / 32;                       // 16-byte chunks per row
  const int64_t per_pass = (int64_t)G * CPL;
  const int npass = (int)((C + per_pass - 1) / per_pass);
  const int lane = threadIdx.x & 31;
  const int li = lane % G;                        // lane within its group
  const int64_t groups_per_block = (kThreads / 32) * (32 / G);
  const int64_t gid = blockIdx.x * groups_per_block + (threadIdx.x >> 5) * (32 / G) + lane / G;
  const int64_t ngroups = (int64_t)gridDim.x * groups_per_block;
  const int64_t total = pb.P * N;
  const int64_t begin = total * gid / ngroups;
  const int64_t end = total * (gid + 1) / ngroups;
  const int64_t my_n = end - begin;

  // x of the current routed row as fp32 pairs (pass 0); reloaded when p changes
  uint64_t xr[CPL][16];
  int64_t xp = -1;
  auto load_x = [&](int64_t p, int pass) {
    const int32_t tok = token_of_row(pb.row_to_token, (int32_t)p, pb.T, pb.err);
    const uint4* xs = reinterpret_cast<const uint4*>(pb.x + (int64_t)tok * K);
#pragma unroll
    for (int i = 0; i < CPL; ++i) {
      const int64_t ch = pass * per_pass + (int64_t)i * G + li;
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        uint4 q = make_uint4(0, 0, 0, 0);
        if (ch < C) q = __ldg(xs + ch * 4 + v);
        const uint32_t w4[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
        for (int j = 0; j < 4; ++j)
          xr[i][v * 4 + j] = pack2(__uint_as_float(w4[j] << 16),
                                   __uint_as_float(w4[j] & 0xFFFF0000u));
      }
    }
  };
  // The first routed row's activations do not depend on the offsets: start
  // loading them before the prologue barrier.
  if (my_n > 0 && npass == 1) {
    xp = begin / N;
    load_x(xp, 0);
  }

  // pair table: entry b -> (value of even element, value of odd element),
  // one 8-byte column per lane; 16-byte stores fill two columns at once.
  // Filled from constant memory while the offsets load.
  for (int i = threadIdx.x; i < 256 * 16; i += kThreads) {
    const uint32_t b = (uint32_t)i >> 4;
    const uint32_t qe = (F == Fmt::NF4) ? (b >> 4) : (b & 15u);
    const uint32_t qo = (F == Fmt::NF4) ? (b & 15u) : (b >> 4);
    const uint32_t lo = __float_as_uint(code_value(F, qe)), hi = __float_as_uint(code_value(F, qo));
    *reinterpret_cast<uint4*>(smem + b * 256 + (i & 15) * 16) = make_uint4(lo, hi, lo, hi);
  }
  load_offsets_clamped(pb.offsets, pb.E, pb.P, off_s, pb.err);  // barrier inside

  const uint64_t* lut = reinterpret_cast<const uint64_t*>(smem);
  const uint32_t lanebits = (uint32_t)lane << 3;  // this lane's table column

  uint4 pk[D][CPL];
  float sc[D][CPL];
  auto issue = [&](int d, const TaskCursor& c, int pass) {
    const int64_t wrow = (int64_t)c.e * N + c.n;
    const uint4* src = reinterpret_cast<const uint4*>(pb.w + wrow * (K / 2));
#pragma unroll
    for (int i = 0; i < CPL; ++i) {
      const int64_t ch = pass * per_pass + (int64_t)i * G + li;
      if (ch < C) {
        pk[d][i] = __ldg(src + ch);
        sc[d][i] = chunk_scale<F>(pb.scale, wrow, K, ch);
      } else {
        pk[d][i] = make_uint4(0x77777777u, 0x77777777u, 0x77777777u, 0x77777777u);
        sc[d][i] = 0.0f;
      }
    }
  };
  // sum_k value(code_k) * x_k over one 16-byte chunk, four independent
  // fp32x2 accumulators (one per packed word), then times the block scale
  auto dot = [&](const uint4 (&q)[CPL], const float (&s)[CPL]) {
    float acc = 0.0f;
#pragma unroll
    for (int i = 0; i < CPL; ++i) {
      const uint32_t w4[4] = {q[i].x, q[i].y, q[i].z, q[i].w};
      uint64_t a2[4] = {0, 0, 0, 0};
#pragma unroll
      for (int b = 0; b < 4; ++b) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint32_t off = prmt(w4[j], lanebits, 0x5504u | (b << 4));
          a2[j] = fma2(lut[off >> 3], xr[i][j * 4 + b], a2[j]);
        }
      }
      const float part = (sum2(a2[0]) + sum2(a2[1])) + (sum2(a2[2]) + sum2(a2[3]));
      acc = fmaf(part, s[i], acc);
    }
    return acc;
  };

  // Whole warps run the loop the same number of times (shuffles inside).
  int64_t max_n = my_n;
#pragma unroll
  for (int o = G; o < 32; o <<= 1)
    max_n = max(max_n, __shfl_xor_sync(0xffffffffu, max_n, o));

  TaskCursor cc, ci;  // compute cursor, issue cursor
  if (my_n > 0) {
    cc.start(begin, N, off_s, pb.E);
    ci = cc;
  }
  if (npass == 1) {
#pragma unroll
    for (int d = 0; d < D; ++d)
      if (d < my_n) { issue(d, ci, 0); ci.next(N, off_s, pb.E); }
    for (int64_t i0 = 0; i0 < max_n; i0 += D) {
#pragma unroll
      for (int d = 0; d < D; ++d) {
        const int64_t i = i0 + d;
        const bool live = i < my_n;
        float acc = 0.0f;
        if (live) {
          if (cc.p != xp) { load_x(cc.p, 0); xp = cc.p; }
          acc = dot(pk[d], sc[d]);
          if (i + D < my_n) { issue(d, ci, 0); ci.next(N, off_s, pb.E); }
        }
        if (i < max_n) {
#pragma unroll
          for (int o = G / 2; o; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o, G);
          if (live) {
            if (li == 0) pb.out[cc.p * N + cc.n] = __bfloat16_as_ushort(__float2bfloat16_rn(acc));
            cc.next(N, off_s, pb.E);
          }
        }
      }
    }
  } else {
    // Rows longer than one pass: x is reloaded per pass, no prefetch.
    for (int64_t i = 0; i < max_n; ++i) {
      const bool live = i < my_n;
      float acc = 0.0f;
      if (live) {
        for (int pass = 0; pass < npass; ++pass) {
          load_x(cc.p, pass);
          issue(0, cc, pass);
          acc += dot(pk[0], sc[0]);
        }
      }
#pragma unroll
      for (int o = G / 2; o; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o, G);
      if (live) {
        if (li == 0) pb.out[cc.p * N + cc.n] = __bfloat16_as_ushort(__float2bfloat16_rn(acc));
        cc.next(N, off_s, pb.E);
      }
    }
  }
}

template <Fmt F, int G, int CPL>
cudaError_t launch_gc(const GroupedProblem& pb, int num_sms, cudaStream_t s) {
  constexpr int D = CPL == 1 ? 12 : (CPL == 2 ? 7 : 2);
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
    if (cpl > 3) { npass = (C + 3 * G - 1) / (3 * G); cpl = 3; }
    const int64_t idle = npass * cpl * G - C;
    if (idle < best_idle) { best_idle = idle; bestG = G; bestCPL = (int)cpl; }
  }
#define GBW_GEMV_CASE(GG, CC) \
  if (bestG == GG && bestCPL == CC) return launch_gc<F, GG, CC>(pb, num_sms, s);
  GBW_GEMV_CASE(32, 1) GBW_GEMV_CASE(32, 2) GBW_GEMV_CASE(32, 3)
  GBW_GEMV_CASE(16, 1) GBW_GEMV_CASE(16, 2) GBW_GEMV_CASE(16, 3)
  GBW_GEMV_CASE(8, 1) GBW_GEMV_CASE(8, 2) GBW_GEMV_CASE(8, 3)
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
