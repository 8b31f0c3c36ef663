// gemv.cu -- bandwidth-targeted grouped GEMV for decode-sized batches.
//
// "grouped-nf4-gemm 0.43.0", release notes at the top of the page: on GPUs
// with many SMs, single-request decode at Qwen3-30B-A3B's expert shapes uses
// a bandwidth-targeted GEMV instead of the tensor-core GEMM.  With one
// routed row per expert every weight byte is used once, so the kernel is
// bound by HBM and never touches the tensor cores.
//
// B200 design (one CTA of 12 warps per SM):
//   work   the P*N weight rows (routed row p, output column n) are cut into
//          row groups of RG rows (G lanes per row, RG = 32 / G); each CTA
//          takes a contiguous range of groups and each warp a contiguous
//          chunk of it;
//   loads  a warp issues the 16-byte loads of its rows' codes and scales for
//          up to MG groups at once, straight into registers, so a CTA has
//          its whole decode-sized share in flight about a microsecond after
//          it starts, with no barrier, producer or staging copy in between;
//   decode one packed byte (two codes) is decoded by one 4-byte shared-
//          memory lookup that returns both codebook values as bf16, from a
//          table holding one column per lane (entry b of lane l at
//          b*256 + l*4, so the 32 lookups of a warp never share a bank; the
//          table sits at a 64 KB-aligned shared address, so one byte permute
//          builds the whole address), multiplied into fp32 accumulators by
//          fma.rn.f32.bf16 with the bf16 activations (the product of two
//          bf16 values is exact in fp32);
//   reduce each 16-byte unit's partial sum is scaled by its block scale; the
//          G lanes of a row reduce with shuffles, two rows at a time (the
//          lanes first swap halves, so a pair costs one shuffle more than a
//          single row).
// Numerics: MXFP4 codes are exact in bf16, so the products are exact.  NF4
// codebook values are rounded to bf16 once (relative error <= 2^-9), and
// the absmax multiplies the partial sum in fp32; the result stays well
// inside |gpu - exact| <= 1e-2 * rms(row) (the stated tolerance).
#include <algorithm>
#include <mutex>

#include "common.cuh"

namespace gbw {
namespace {

constexpr int kThreads = 384;  // 12 warps: up to 168 registers a thread
constexpr int kWarps = kThreads / 32;
constexpr int kLutBytes = 256 * 256;  // 256 entries x 256-byte rows

// Codebook value of code q, from immediates (a select tree, no memory
// access: a table in constant memory costs a cold miss on every launch).
// NF4: the 16 QLoRA levels; MXFP4: OCP e2m1 (bit 3 = sign).
__device__ __forceinline__ float code_value(Fmt F, uint32_t q) {
  if (F == Fmt::NF4) {
    const float lo8[8] = {-1.0f, -0.6961928009986877f, -0.5250730514526367f,
                          -0.39491748809814453f, -0.28444138169288635f,
                          -0.18477343022823334f, -0.09105003625154495f, 0.0f};
    const float hi8[8] = {0.07958029955625534f, 0.16093020141124725f,
                          0.24611230194568634f, 0.33791524171829224f,
                          0.44070982933044434f, 0.5626170039176941f,
                          0.7229568362236023f, 1.0f};
    float r = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      r = (q == (uint32_t)i) ? lo8[i] : r;
      r = (q == (uint32_t)(i + 8)) ? hi8[i] : r;
    }
    return r;
  }
  const uint32_t m = q & 7u;
  // e2m1 magnitude: exponent field m >> 1 (bias 1), mantissa bit m & 1
  const float mag = (m < 2u) ? 0.5f * (float)m
                             : __int_as_float((int)((126u + (m >> 1)) << 23)) *
                                   (1.0f + 0.5f * (float)(m & 1u));
  return (q & 8u) ? -mag : mag;
}

__device__ __forceinline__ float e8m0_f32(uint32_t s) {
  if (s == 0xFFu) return __int_as_float(0x7FC00000);
  if (s == 0u) return __int_as_float(0x00400000);  // 2^-127
  return __int_as_float((int)(s << 23));
}

__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}

// a0 += lo(w) * lo(x), a1 += hi(w) * hi(x): bf16 inputs, fp32 accumulate.
__device__ __forceinline__ void fma_pair(float& a0, float& a1, uint32_t w,
                                         uint32_t x) {
  asm("{\n .reg .b16 wl, wh, xl, xh;\n"
      " mov.b32 {wl, wh}, %2;\n"
      " mov.b32 {xl, xh}, %3;\n"
      " fma.rn.f32.bf16 %0, wl, xl, %0;\n"
      " fma.rn.f32.bf16 %1, wh, xh, %1;\n}\n"
      : "+f"(a0), "+f"(a1)
      : "r"(w), "r"(x));
}

// sum over the 32 weights of one 16-byte unit of code value * x.  Byte m of
// the unit holds elements 2m, 2m+1, and x pair m holds the same elements.
__device__ __forceinline__ float dot_unit(const uint4& q, const uint32_t (&x)[16],
                                          uint32_t lut_lane) {
  const uint32_t w[4] = {q.x, q.y, q.z, q.w};
  float a[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int m = 0; m < 16; ++m) {
    // table base | byte << 8 | lane*4: the lane's column of that byte's entry
    const uint32_t addr = prmt(w[m >> 2], lut_lane, 0x7604u | ((m & 3) << 4));
    const uint32_t v = lds32(addr);
    fma_pair(a[2 * (m & 3)], a[2 * (m & 3) + 1], v, x[m]);
  }
  return ((a[0] + a[1]) + (a[2] + a[3])) + ((a[4] + a[5]) + (a[6] + a[7]));
}

// Shared window: the decode table at the first 64 KB-aligned address; the
// clamped expert offsets below it when they fit there, else after it.
struct Layout {
  uint32_t lut, off;
};

__device__ __forceinline__ Layout make_layout(uint32_t s0, int32_t E) {
  Layout L;
  L.lut = (s0 + 0xFFFFu) & ~0xFFFFu;
  const uint32_t ob = 4u * (uint32_t)(E + 1);
  const uint32_t lo = (s0 + 15u) & ~15u;
  L.off = lo + ob <= L.lut ? lo : L.lut + (uint32_t)kLutBytes;
  return L;
}

// Row groups a warp loads per round (register budget for codes + scales).
template <int UPL>
struct Round {
  static constexpr int MG = UPL == 1 ? 12 : (UPL == 2 ? 7 : 5);
};

template <Fmt F, int G, int UPL>
__global__ void __launch_bounds__(kThreads, 1)
gemv_kernel(const GroupedProblem pb, const int64_t ngroups, const int npass) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  const Layout lay = make_layout(smem_u32(smem_raw), pb.E);
  uint8_t* const base = smem_raw - smem_u32(smem_raw);  // shared window start
  int32_t* off_s = reinterpret_cast<int32_t*>(base + lay.off);

  constexpr int RG = 32 / G;                // rows per row group
  constexpr int MG = Round<UPL>::MG;        // row groups per load round
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int li = lane % G, rs = lane / G;
  const int64_t K = pb.K, N = pb.N;
  const int64_t U = K / 32;                 // 16-byte units per row
  const int64_t srow = (F == Fmt::NF4) ? K / 64 : K / 32;  // scales per row

  // this warp's row groups: a contiguous chunk of the CTA's contiguous range
  const int64_t c0 = ngroups * blockIdx.x / gridDim.x;
  const int64_t c1 = ngroups * (blockIdx.x + 1) / gridDim.x;
  const int64_t g0 = c0 + (c1 - c0) * warp / kWarps;
  const int64_t g1 = c0 + (c1 - c0) * (warp + 1) / kWarps;

  // walk state: routed row p and column n of the next row group (advanced
  // by carry: one division per warp)
  int32_t p = (int32_t)(g0 * RG / N);
  int64_t n = g0 * RG - (int64_t)p * N;

  uint32_t xr[UPL][16];
  int64_t xkey = -1;  // token * npass + pass held in xr
  auto load_x = [&](int32_t tok, int pass) {
    const uint4* xs = reinterpret_cast<const uint4*>(pb.x + (int64_t)tok * K);
#pragma unroll
    for (int i = 0; i < UPL; ++i) {
      const int64_t u = ((int64_t)pass * UPL + i) * G + li;
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        uint4 q = make_uint4(0u, 0u, 0u, 0u);
        if (u < U) q = __ldg(xs + u * 4 + v);
        xr[i][4 * v] = q.x;
        xr[i][4 * v + 1] = q.y;
        xr[i][4 * v + 2] = q.z;
        xr[i][4 * v + 3] = q.w;
      }
    }
    xkey = (int64_t)tok * npass + pass;
  };
  // Programmatic dependent launch.  x may be written by the kernel launched
  // just before this one, so it is read only after grid_dependency_wait;
  // with GBW_FLAG_OVERLAP_PREV the offsets, row map, codes and scales are
  // not, so they are read while that kernel finishes.  The next kernel may
  // launch once this one has passed its wait.
  const bool early = (pb.flags & GBW_FLAG_OVERLAP_PREV) != 0;
  bool waited = false;
  auto ready = [&]() {
    if (!waited) {
      grid_dependency_wait();
      grid_launch_dependents();
      waited = true;
    }
  };
  if (!early) ready();
  // independent global loads first (the offsets and the first row's token),
  // so the table below is built while they are in flight
  const OffsetRegs offr = prefetch_offsets(pb.offsets, pb.E);
  int32_t tok = g0 < g1 ? token_of_row(pb.row_to_token, p, pb.T, pb.err) : 0;
  // pair table: entry b -> bf16 (value of the even element, value of the odd
  // element) in every lane's column.  Thread b < 256 builds entry b and
  // writes its 128-byte row with eight 16-byte stores, starting at chunk
  // b % 8 so the 32 stores of a warp instruction spread over all banks.
  // It touches no caller memory.
  if (threadIdx.x < 256) {
    const uint32_t b = threadIdx.x;
    const uint32_t qe = (F == Fmt::NF4) ? (b >> 4) : (b & 15u);
    const uint32_t qo = (F == Fmt::NF4) ? (b & 15u) : (b >> 4);
    const uint32_t v =
        (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(code_value(F, qe))) |
        ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(code_value(F, qo))) << 16);
    uint8_t* row = base + lay.lut + b * 256;
#pragma unroll
    for (int c = 0; c < 8; ++c)
      *reinterpret_cast<uint4*>(row + ((c + b) & 7u) * 16) = make_uint4(v, v, v, v);
  }
  if (!early && g0 < g1) load_x(tok, 0);
  commit_offsets(offr, pb.offsets, pb.E, pb.P, off_s, pb.err);  // barrier inside

  if (g0 >= g1) ready();
  const uint32_t lut_lane = lay.lut | ((uint32_t)lane * 4u);
  int32_t e = g0 < g1 ? expert_of_row(off_s, pb.E, p) : 0;
  const bool hi = (li & (G / 2)) != 0;
  for (int64_t g = g0; g < g1;) {
    // one round: up to MG row groups of one routed row (one x)
    int cnt = (int)min((int64_t)MG, g1 - g);
    cnt = (int)min((int64_t)cnt, (N - n) / RG);
    const int64_t wrow0 = (int64_t)e * N + n + rs;  // weight row of group 0
    float acc[MG];
#pragma unroll
    for (int k = 0; k < MG; ++k) acc[k] = 0.0f;
    for (int pass = 0; pass < npass; ++pass) {
      uint4 q[MG][UPL];
      float sc[MG][UPL];
#pragma unroll
      for (int k = 0; k < MG; ++k) {
        const int64_t wrow = wrow0 + (int64_t)k * RG;
#pragma unroll
        for (int i = 0; i < UPL; ++i) {
          const int64_t u = ((int64_t)pass * UPL + i) * G + li;
          q[k][i] = make_uint4(0u, 0u, 0u, 0u);
          sc[k][i] = 0.0f;
          if (k < cnt && u < U) {
            q[k][i] = __ldg(reinterpret_cast<const uint4*>(pb.w + wrow * (K / 2)) + u);
            if (F == Fmt::NF4)
              sc[k][i] = __ldg(reinterpret_cast<const float*>(pb.scale) + wrow * srow + (u >> 1));
            else
              sc[k][i] = e8m0_f32(__ldg(reinterpret_cast<const uint8_t*>(pb.scale) + wrow * srow + u));
          }
        }
      }
      if ((int64_t)tok * npass + pass != xkey) {
        ready();
        load_x(tok, pass);
      }
#pragma unroll
      for (int k = 0; k < MG; ++k)
#pragma unroll
        for (int i = 0; i < UPL; ++i)
          if (k < cnt) acc[k] = fmaf(dot_unit(q[k][i], xr[i], lut_lane), sc[k][i], acc[k]);
    }
    // Reduce pairs of row groups over the G lanes: the lower half of the
    // lanes collects group 2m, the upper half group 2m + 1.
#pragma unroll
    for (int m = 0; m < (MG + 1) / 2; ++m) {
      if (2 * m < cnt) {
        const float a0 = acc[2 * m], a1 = 2 * m + 1 < MG ? acc[2 * m + 1] : 0.0f;
        float keep = hi ? a1 : a0;
        keep += __shfl_xor_sync(0xffffffffu, hi ? a0 : a1, G / 2, G);
#pragma unroll
        for (int o = G / 4; o; o >>= 1) keep += __shfl_xor_sync(0xffffffffu, keep, o, G);
        const int k = 2 * m + (hi ? 1 : 0);
        if ((li & (G / 2 - 1)) == 0 && k < cnt)
          pb.out[(int64_t)p * N + n + (int64_t)k * RG + rs] =
              __bfloat16_as_ushort(__float2bfloat16_rn(keep));
      }
    }
    // advance
    g += cnt;
    n += (int64_t)cnt * RG;
    if (n == N && g < g1) {
      n = 0;
      ++p;
      e = expert_of_row(off_s, pb.E, p);
      tok = token_of_row(pb.row_to_token, p, pb.T, pb.err);
    }
  }
}

struct Shape {
  int G, UPL, npass;
};

// Lanes per row G and units per lane UPL with the fewest idle unit slots;
// rows longer than 32 * 3 units take several passes.
Shape pick_shape(int64_t U) {
  Shape best{32, 3, (int)((U + 95) / 96)};
  if (U > 96) return best;
  int64_t best_idle = INT64_MAX;
  for (int G : {32, 16, 8})
    for (int upl : {1, 2, 3})
      if ((int64_t)G * upl >= U) {
        const int64_t idle = (int64_t)G * upl - U;
        if (idle < best_idle) { best_idle = idle; best = Shape{G, upl, 1}; }
      }
  return best;
}

// Dynamic shared memory: enough that a 64 KB-aligned 64 KB table fits
// wherever the window starts, plus the offsets.
size_t gemv_smem(int32_t E) {
  return 2 * (size_t)kLutBytes + 4 * (size_t)(E + 1) + 64;
}

// Per-device, per-kernel opt-in to the kernel's dynamic shared memory.
// Guarded by a mutex: host threads may launch concurrently.
cudaError_t opt_in(const void* fn, size_t smem) {
  struct Entry { const void* fn; int dev; size_t smem; };
  static std::mutex mu;
  static Entry done[256];
  static int ndone = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  for (int i = 0; i < ndone; ++i)
    if (done[i].fn == fn && done[i].dev == dev && done[i].smem >= smem) return cudaSuccess;
  e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  for (int i = 0; i < ndone; ++i)
    if (done[i].fn == fn && done[i].dev == dev) {
      done[i].smem = smem;
      return cudaSuccess;
    }
  if (ndone < 256) done[ndone++] = Entry{fn, dev, smem};
  return cudaSuccess;
}

template <Fmt F, int G, int UPL>
cudaError_t launch_t(const GroupedProblem& pb, int64_t ngroups, int npass,
                     int grid, cudaStream_t s) {
  auto k = gemv_kernel<F, G, UPL>;
  const size_t smem = gemv_smem(pb.E);
  cudaError_t e = opt_in(reinterpret_cast<const void*>(k), smem);
  if (e != cudaSuccess) return e;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, k, pb, ngroups, npass);
}

template <Fmt F>
cudaError_t launch_f(const GroupedProblem& pb, const Shape& sh, int64_t ngroups,
                     int grid, cudaStream_t s) {
#define GBW_GEMV_CASE(GG, UU) \
  if (sh.G == GG && sh.UPL == UU) return launch_t<F, GG, UU>(pb, ngroups, sh.npass, grid, s);
  GBW_GEMV_CASE(32, 1) GBW_GEMV_CASE(32, 2) GBW_GEMV_CASE(32, 3)
  GBW_GEMV_CASE(16, 1) GBW_GEMV_CASE(16, 2) GBW_GEMV_CASE(16, 3)
  GBW_GEMV_CASE(8, 1) GBW_GEMV_CASE(8, 2) GBW_GEMV_CASE(8, 3)
#undef GBW_GEMV_CASE
  return cudaErrorInvalidValue;
}

}  // namespace

bool gemv_fits(Fmt, const GroupedProblem& pb, int) {
  return gemv_smem(pb.E) <= 227 * 1024;
}

cudaError_t launch_gemv(Fmt f, const GroupedProblem& pb, int num_sms,
                        cudaStream_t s) {
  if (pb.P == 0 || pb.N == 0) return cudaSuccess;
  const Shape sh = pick_shape(pb.K / 32);
  const int64_t ngroups = pb.P * (pb.N / (32 / sh.G));
  const int grid = (int)std::min<int64_t>(num_sms, (ngroups + kWarps - 1) / kWarps);
  return f == Fmt::NF4 ? launch_f<Fmt::NF4>(pb, sh, ngroups, grid, s)
                       : launch_f<Fmt::MXFP4>(pb, sh, ngroups, grid, s);
}

}  // namespace gbw
