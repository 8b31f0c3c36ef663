// gemv.cu -- bandwidth-targeted grouped GEMV for decode-sized batches.
//
// "grouped-nf4-gemm 0.43.0", release notes at the top of the page: on GPUs
// with many SMs, single-request decode at Qwen3-30B-A3B's expert shapes uses
// a bandwidth-targeted GEMV instead of the tensor-core GEMM.  With one
// routed row per expert every weight byte is used once, so the kernel is
// bound by HBM and never touches the tensor cores.
//
// B200 design (two CTAs of 8 warps per SM, 128 registers a thread; a warp's
// share of a decode-sized launch fits one round of loads):
//   work   the P*N weight rows (routed row p, output column n) are cut into
//          row groups of RG rows (G lanes per row, RG = 32 / G); each CTA
//          takes a contiguous range of groups and each warp a contiguous
//          chunk of it;
//   loads  a warp issues the 16-byte loads of its rows' codes and scales for
//          up to MG row groups at once, straight into registers, so a CTA has
//          its whole decode-sized share in flight about a microsecond after
//          it starts, with no barrier, producer or staging copy in between.
//          Addresses come from one 64-bit row pointer per round plus
//          constant strides (the per-load 64-bit index arithmetic used to
//          cost as many instructions as the decode itself);
//   decode one packed byte (two codes) is decoded by one 4-byte shared-memory
//          lookup that returns both codebook values as bf16, from a table
//          holding one column per lane (entry b of lane l at b*256 + l*4, so
//          the 32 lookups of a warp never share a bank).  The offset is one
//          byte permute and the table's base an immediate of the load, and
//          each value is multiplied into an fp32 accumulator by
//          fma.rn.f32.bf16 with the bf16 activation (one instruction; the
//          product of two bf16 values is exact in fp32).  Measured on B200
//          with the data in registers: 76 instructions per 16-byte unit, 40
//          weights per clock per SM -- the rate HBM delivers NF4 weights;
//   reduce each 16-byte unit's partial sum is scaled by its block scale; the
//          G lanes of a row reduce with shuffles, two rows at a time (the
//          lanes first swap halves, so a pair costs one shuffle more than a
//          single row).
// SwiGLU variant (the gate_up projection of the fused expert pass at decode
// sizes, G = 32): virtual row 2j of a routed row is gate row j and 2j + 1 is
// up row I + j, so a round's groups pair up; the pair reduction leaves the
// gate total in the lower half of the lanes and the up total in the upper
// half, and one more shuffle lets lane 0 write h = bf16(silu(bf16 gate) *
// bf16 up) to h [P, I].
// Numerics: MXFP4 codes are exact in bf16, so the products are exact.  NF4
// codebook values are rounded to bf16 once (relative error <= 2^-9), and
// the absmax multiplies the partial sum in fp32; the result stays well
// inside |gpu - exact| <= 1e-2 * rms(row) (the stated tolerance).
#include <algorithm>
#include <mutex>

#include "common.cuh"

namespace gbw {
namespace {

constexpr int kThreads = 256;  // 8 warps, <= 128 registers: two CTAs per SM
constexpr int kWarps = kThreads / 32;
constexpr int kLutBytes = 256 * 256;  // 256 entries x 256-byte rows (lanes use 128 bytes)
// Shared-window offset of the dynamic shared memory of a kernel without
// static shared memory (measured on B200).  The table starts there; a launch
// that finds it elsewhere adds the base at run time (one more instruction
// per lookup).
constexpr uint32_t kLutBaseGuess = 1024;
constexpr uint32_t kRuntimeBase = 0xFFFFFFFFu;

// bf16 bits of the codebook value of code q, from immediates (a select
// tree on the bits of q, no memory access: a table in constant memory costs
// a cold miss on every launch).  Word j holds the values of codes 2j (low
// half) and 2j + 1.  NF4: bf16_rn of the 16 QLoRA levels (-1, -0.6961928,
// -0.5250731, -0.3949175, -0.2844414, -0.1847734, -0.0910500, 0, 0.0795803,
// 0.1609302, 0.2461123, 0.3379152, 0.4407098, 0.5626170, 0.7229568, 1);
// MXFP4: the e2m1 values 0, 0.5, 1, 1.5, 2, 3, 4, 6 and their negatives
// (bit 3 = sign, code 8 = -0), exact in bf16.
__device__ __forceinline__ uint32_t code_bf16(Fmt F, uint32_t q) {
  const bool nf4 = F == Fmt::NF4;
  const uint32_t w0 = nf4 ? 0xbf32bf80u : 0x3f000000u, w1 = nf4 ? 0xbecabf06u : 0x3fc03f80u;
  const uint32_t w2 = nf4 ? 0xbe3dbe92u : 0x40404000u, w3 = nf4 ? 0x0000bdbau : 0x40c04080u;
  const uint32_t w4 = nf4 ? 0x3e253da3u : 0xbf008000u, w5 = nf4 ? 0x3ead3e7cu : 0xbfc0bf80u;
  const uint32_t w6 = nf4 ? 0x3f103ee2u : 0xc040c000u, w7 = nf4 ? 0x3f803f39u : 0xc0c0c080u;
  const uint32_t j = q >> 1;
  const uint32_t a = (j & 1u) ? w1 : w0, b = (j & 1u) ? w3 : w2;
  const uint32_t c = (j & 1u) ? w5 : w4, d = (j & 1u) ? w7 : w6;
  const uint32_t e = (j & 2u) ? b : a, f = (j & 2u) ? d : c;
  const uint32_t w = (j & 4u) ? f : e;
  return (q & 1u) ? (w >> 16) : (w & 0xFFFFu);
}

__device__ __forceinline__ float e8m0_f32(uint32_t s) {
  if (s == 0xFFu) return __int_as_float(0x7FC00000);
  if (s == 0u) return __int_as_float(0x00400000);  // 2^-127
  return __int_as_float((int)(s << 23));
}

// One table entry (two bf16 values): `off` = entry * 256 + lane * 4.
template <uint32_t kBase>
__device__ __forceinline__ uint32_t lut_ld(uint32_t off, uint32_t base) {
  uint32_t v;
  if (kBase != kRuntimeBase)
    asm volatile("ld.shared.b32 %0, [%1+%2];" : "=r"(v) : "r"(off), "n"(kBase));
  else
    asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(off + base));
  return v;
}

// a0 += lo(w) * lo(x), a1 += hi(w) * hi(x): bf16 inputs, fp32 accumulate
// (one instruction each).
__device__ __forceinline__ void fma_pair(float& a0, float& a1, uint32_t w, uint32_t x) {
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
template <uint32_t kBase>
__device__ __forceinline__ float dot_unit(const uint4& q, const uint32_t (&x)[16],
                                          uint32_t lane4, uint32_t base) {
  const uint32_t w[4] = {q.x, q.y, q.z, q.w};
  // four fp32 chains of eight FMAs; a warp's units are independent, so the
  // chains of several units interleave
  float a[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int m = 0; m < 16; ++m)  // byte << 8 | lane * 4: the lane's column of that byte's entry
    fma_pair(a[2 * (m & 1)], a[2 * (m & 1) + 1],
             lut_ld<kBase>(prmt(w[m >> 2], lane4, 0x7604u | ((m & 3) << 4)), base), x[m]);
  return (a[0] + a[1]) + (a[2] + a[3]);
}

// Row groups a warp loads per round (register budget for codes + scales,
// within 128 registers a thread).
template <Fmt F, int UPL>
struct Round {
  static constexpr int MG = UPL == 1 ? 10 : (UPL == 2 ? 6 : (F == Fmt::NF4 ? 2 : 3));
};

// The row groups [g0, g1) of one warp, after the kernel's prologue.
template <Fmt F, int G, int UPL, bool kGLU, uint32_t kBase>
__device__ __forceinline__ void gemv_main(const GroupedProblem& pb, const int32_t* off_s,
                                          int64_t g0, int64_t g1, int npass, int32_t tok,
                                          uint32_t base, bool waited) {
  static_assert(!kGLU || G == 32, "the SwiGLU variant takes one row per group");
  constexpr int RG = 32 / G;                // rows per row group
  // row groups per load round (even for SwiGLU: gate/up pairs)
  constexpr int MG = kGLU ? (Round<F, UPL>::MG & ~1) : Round<F, UPL>::MG;
  const int lane = threadIdx.x & 31;
  const int li = lane % G, rs = lane / G;
  const int64_t K = pb.K, N = pb.N;
  const int32_t U = (int32_t)(K / 32);      // 16-byte units per row
  const int32_t srow = (int32_t)((F == Fmt::NF4) ? K / 64 : K / 32);  // scales per row
  const int64_t wstride = (int64_t)RG * U;  // 16-byte units between row groups
  const int64_t sstride = (int64_t)RG * srow;
  const uint32_t lane4 = (uint32_t)lane * 4u;
  const uint4* const w16 = reinterpret_cast<const uint4*>(pb.w);

  // walk state: routed row p and column n of the next row group (advanced
  // by carry: one division per warp)
  int32_t p = (int32_t)(g0 * RG / N);
  int64_t n = g0 * RG - (int64_t)p * N;
  int32_t e = expert_of_row(off_s, pb.E, p);

  uint32_t xr[UPL][16];  // x of the current row and pass (bf16 pairs)
  int64_t xkey = -1;     // token * npass + pass held in xr
  const bool hi = (li & (G / 2)) != 0;
  for (int64_t g = g0; g < g1;) {
    // one round: up to MG row groups of one routed row (one x)
    int cnt = (int)min((int64_t)MG, g1 - g);
    cnt = (int)min((int64_t)cnt, (N - n) / RG);
    // weight row of group 0; SwiGLU: gate rows from wp, up rows from wpu
    // (group k is gate or up row (n + k) / 2)
    const int64_t I = N / 2;
    const int64_t wrow0 = kGLU ? (int64_t)e * N + n / 2 : (int64_t)e * N + n + rs;
    const uint4* const wp = w16 + wrow0 * U;
    const uint4* const wpu = w16 + (wrow0 + I) * U;
    const int64_t s0 = wrow0 * srow, s0u = (wrow0 + I) * srow;
    float acc[MG];
#pragma unroll
    for (int k = 0; k < MG; ++k) acc[k] = 0.0f;
    for (int pass = 0; pass < npass; ++pass) {
      int32_t uo[UPL];  // this lane's units in the pass (>= U: past the row)
#pragma unroll
      for (int i = 0; i < UPL; ++i) uo[i] = (pass * UPL + i) * G + li;
      uint4 q[MG][UPL];
      uint32_t sc[MG][UPL];  // raw scale bits, converted when used
#pragma unroll
      for (int k = 0; k < MG; ++k)
#pragma unroll
        for (int i = 0; i < UPL; ++i) {
          q[k][i] = make_uint4(0u, 0u, 0u, 0u);
          sc[k][i] = 0u;
          if (k < cnt && uo[i] < U) {
            const uint4* rp = kGLU ? ((k & 1) ? wpu : wp) + (int64_t)(k >> 1) * U : wp + k * wstride;
            const int64_t so = kGLU ? ((k & 1) ? s0u : s0) + (int64_t)(k >> 1) * srow : s0 + k * sstride;
            q[k][i] = __ldg(rp + uo[i]);
            if (F == Fmt::NF4)
              sc[k][i] = __ldg(reinterpret_cast<const uint32_t*>(pb.scale) + so + (uo[i] >> 1));
            else
              sc[k][i] = __ldg(reinterpret_cast<const uint8_t*>(pb.scale) + so + uo[i]);
          }
        }
      if ((int64_t)tok * npass + pass != xkey) {
        // x may be written by the kernel launched just before this one: it
        // is read only after that kernel has completed
        if (!waited) {
          grid_dependency_wait();
          grid_launch_dependents();
          waited = true;
        }
        const uint4* xs = reinterpret_cast<const uint4*>(pb.x + (int64_t)tok * K);
#pragma unroll
        for (int i = 0; i < UPL; ++i)
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            uint4 t = make_uint4(0u, 0u, 0u, 0u);
            if (uo[i] < U) t = __ldg(xs + uo[i] * 4 + v);
            xr[i][4 * v] = t.x;
            xr[i][4 * v + 1] = t.y;
            xr[i][4 * v + 2] = t.z;
            xr[i][4 * v + 3] = t.w;
          }
        xkey = (int64_t)tok * npass + pass;
      }
#pragma unroll
      for (int k = 0; k < MG; ++k)
#pragma unroll
        for (int i = 0; i < UPL; ++i)
          if (k < cnt) {
            const float s = F == Fmt::NF4 ? __uint_as_float(sc[k][i]) : e8m0_f32(sc[k][i]);
            acc[k] = fmaf(dot_unit<kBase>(q[k][i], xr[i], lane4, base), s, acc[k]);
          }
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
        if (kGLU) {
          // lower half: gate total of h column (n / 2 + m); upper half: up
          const float g = __bfloat162float(__float2bfloat16_rn(keep));
          const float u = __shfl_xor_sync(0xffffffffu, g, G / 2);
          if (lane == 0)
            pb.out[(int64_t)p * I + n / 2 + m] =
                __bfloat16_as_ushort(__float2bfloat16_rn(g / (1.0f + expf(-g)) * u));
        } else {
          const int k = 2 * m + (hi ? 1 : 0);
          if ((li & (G / 2 - 1)) == 0 && k < cnt)
            pb.out[(int64_t)p * N + n + (int64_t)k * RG + rs] =
                __bfloat16_as_ushort(__float2bfloat16_rn(keep));
        }
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
  if (!waited) {
    grid_dependency_wait();
    grid_launch_dependents();
  }
}

template <Fmt F, int G, int UPL, bool kGLU>
__global__ void __launch_bounds__(kThreads, 2)
gemv_kernel(const GroupedProblem pb, const int64_t ngroups, const int npass) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  const uint32_t base = smem_u32(smem_raw);  // the table: 256 rows of 256 bytes
  int32_t* off_s = reinterpret_cast<int32_t*>(smem_raw + kLutBytes);
  constexpr int RG = 32 / G;
  const int warp = threadIdx.x >> 5;

  // this warp's row groups: a contiguous chunk of the CTA's contiguous range
  // (in gate/up pairs for SwiGLU)
  constexpr int64_t A = kGLU ? 2 : 1;
  const int64_t na = ngroups / A;
  const int64_t c0 = na * blockIdx.x / gridDim.x;
  const int64_t c1 = na * (blockIdx.x + 1) / gridDim.x;
  const int64_t g0 = A * (c0 + (c1 - c0) * warp / kWarps);
  const int64_t g1 = A * (c0 + (c1 - c0) * (warp + 1) / kWarps);

  // Programmatic dependent launch.  Without GBW_FLAG_OVERLAP_PREV every
  // input may come from the kernel launched just before this one, so this
  // kernel waits for it first.  With the flag, the offsets, row map, codes
  // and scales are read while that kernel finishes, and only x waits.  The
  // next kernel may launch once this one has waited.
  const bool early = (pb.flags & GBW_FLAG_OVERLAP_PREV) != 0;
  if (!early) {
    grid_dependency_wait();
    grid_launch_dependents();
  }
  // independent global loads first (the offsets and the first row's token),
  // so the table below is built while they are in flight
  const OffsetRegs offr = prefetch_offsets(pb.offsets, pb.E);
  const int32_t p0 = g0 < g1 ? (int32_t)(g0 * RG / pb.N) : 0;
  const int32_t tok0 = g0 < g1 ? token_of_row(pb.row_to_token, p0, pb.T, pb.err) : 0;
  // pair table: entry b -> bf16 (value of the even element, value of the odd
  // element) in every lane's column.  Thread b < 256 builds entry b and
  // writes its 128-byte row with eight 16-byte stores, starting at chunk
  // b % 8 so the 32 stores of a warp instruction spread over all banks.  It
  // touches no caller memory.
  {
    const uint32_t b = threadIdx.x;  // 256 threads: one entry each
    const uint32_t qe = (F == Fmt::NF4) ? (b >> 4) : (b & 15u);
    const uint32_t qo = (F == Fmt::NF4) ? (b & 15u) : (b >> 4);
    const uint32_t v = code_bf16(F, qe) | (code_bf16(F, qo) << 16);
    uint8_t* row = smem_raw + b * 256;
#pragma unroll
    for (int c = 0; c < 8; ++c)
      *reinterpret_cast<uint4*>(row + ((c + b) & 7u) * 16) = make_uint4(v, v, v, v);
  }
  commit_offsets(offr, pb.offsets, pb.E, pb.P, off_s, pb.err);  // barrier inside

  if (g0 >= g1) {
    if (early) {
      grid_dependency_wait();
      grid_launch_dependents();
    }
    return;
  }
  if (base == kLutBaseGuess)
    gemv_main<F, G, UPL, kGLU, kLutBaseGuess>(pb, off_s, g0, g1, npass, tok0, base, !early);
  else
    gemv_main<F, G, UPL, kGLU, kRuntimeBase>(pb, off_s, g0, g1, npass, tok0, base, !early);
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

// Dynamic shared memory: the 64 KB table, then the offsets.
size_t gemv_smem(int32_t E) { return (size_t)kLutBytes + 4 * (size_t)(E + 1); }

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

template <Fmt F, int G, int UPL, bool kGLU = false>
cudaError_t launch_t(const GroupedProblem& pb, int64_t ngroups, int npass,
                     int grid, cudaStream_t s) {
  auto k = gemv_kernel<F, G, UPL, kGLU>;
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
                        cudaStream_t s, bool glu) {
  if (pb.P == 0 || pb.N == 0) return cudaSuccess;
  const int64_t U = pb.K / 32;
  // SwiGLU: one row per group (G = 32), as many units per lane as the row needs
  const Shape sh = glu ? Shape{32, (int)std::min<int64_t>(3, (U + 31) / 32), (int)((U + 95) / 96)}
                       : pick_shape(U);
  const int64_t ngroups = pb.P * (pb.N / (32 / sh.G));
  // the kernel keys its activation rows as token * npass + pass in 32 bits
  if ((int64_t)std::max<int64_t>(pb.T, pb.P) * sh.npass >= INT32_MAX) return cudaErrorInvalidValue;
  const int grid = (int)std::min<int64_t>(2 * num_sms, (ngroups / (glu ? 2 : 1) + kWarps - 1) / kWarps);
  if (glu) {
#define GBW_GEMV_GLU(FF)                                                              \
  switch (sh.UPL) {                                                                   \
    case 1: return launch_t<FF, 32, 1, true>(pb, ngroups, sh.npass, grid, s);         \
    case 2: return launch_t<FF, 32, 2, true>(pb, ngroups, sh.npass, grid, s);         \
    default: return launch_t<FF, 32, 3, true>(pb, ngroups, sh.npass, grid, s);        \
  }
    if (f == Fmt::NF4) { GBW_GEMV_GLU(Fmt::NF4) } else { GBW_GEMV_GLU(Fmt::MXFP4) }
#undef GBW_GEMV_GLU
  }
  return f == Fmt::NF4 ? launch_f<Fmt::NF4>(pb, sh, ngroups, grid, s)
                       : launch_f<Fmt::MXFP4>(pb, sh, ngroups, grid, s);
}

}  // namespace gbw
