// gemv.cu -- bandwidth-targeted grouped GEMV for decode-sized batches.
//
// "grouped-nf4-gemm 0.43.0", release notes at the top of the page: on GPUs
// with many SMs, single-request decode at Qwen3-30B-A3B's expert shapes uses
// a bandwidth-targeted GEMV instead of the tensor-core GEMM.  With one
// routed row per expert every weight byte is used once, so the kernel is
// bound by HBM and never touches the tensor cores.
//
// B200 design (one persistent CTA per SM, 16 warps):
//   work   the P*N weight rows (routed row p, output column n) are cut into
//          blocks of R consecutive rows of one expert, which are contiguous
//          in memory ([E, N, K/2] codes, [E, N, K/s] scales); each CTA takes a
//          contiguous range of blocks;
//   warp 0 streams its blocks into a shared-memory ring with bulk
//          asynchronous copies (cp.async.bulk, one for the codes and one for
//          the scales of a block), so the bytes in flight do not cost
//          registers: for the decode shapes a CTA's whole share is requested
//          in the first microsecond;
//   warps 1-15 take the staged rows: G lanes per row, each lane owning UPL
//          16-byte units (32 weights) of the row.  One packed byte (two
//          codes) is decoded by one 4-byte shared-memory lookup that returns
//          both codebook values as bf16, from a table holding one column per
//          lane (entry b of lane l at b*256 + l*4, so the 32 lookups of a warp
//          never share a bank; one byte permute builds the address), and
//          multiplied into fp32 accumulators by fma.rn.f32.bf16 with the bf16
//          activations (the product of two bf16 values is exact in fp32).
//          Each unit's partial sum is scaled once by its block scale; the G
//          lanes of a row then reduce with shuffles.
// Numerics: MXFP4 codes are exact in bf16, so the products are exact.  NF4
// codebook values are rounded to bf16 once (relative error <= 2^-9), and
// the absmax multiplies the partial sum in fp32; the result stays well
// inside |gpu - exact| <= 1e-2 * rms(row) (the stated tolerance).
#include <algorithm>

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

constexpr int kThreads = 512;
constexpr int kConsumers = kThreads / 32 - 1;  // warp 0 produces
constexpr int kLutBytes = 256 * 256;           // 256 entries x 256-byte rows
constexpr int kSmemCap = 227 * 1024;           // opt-in shared memory per CTA

struct GemvPlan {
  int64_t nblocks;      // P * N / R
  int32_t R;            // weight rows per block (divides N)
  int32_t npass;        // passes over K (units beyond G*UPL)
  int32_t stage_bytes;  // one ring slot: codes then scales
  int32_t scale_off;    // byte offset of the scales inside a slot
  int32_t nstages;      // ring slots
  int32_t scales_staged;  // 0: scales read from global (unaligned rows)
};

__device__ __forceinline__ float code_value(Fmt F, uint32_t q) {
  if (F == Fmt::NF4) return kNF4g[q];
  const float m = kE2M1g[q & 7u];
  return (q & 8u) ? -m : m;
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

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr));
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

// Shared memory: the decode table sits at the first 64 KB-aligned address of
// the block's window, so a byte permute can place the packed byte into bits
// 8-15 of a table address without an add; the ring slots fill the space
// below and above it.
struct Layout {
  uint32_t lut;        // shared address of the table (64 KB aligned)
  uint32_t meta;       // barriers (2 per slot), abort flag, slot block ids, offsets
  uint32_t low, nlow;  // slots below the table
  uint32_t high;       // slots above the table
  int ns;              // slots in use
  __device__ __forceinline__ uint32_t slot(int i, uint32_t bytes) const {
    return (uint32_t)i < nlow ? low + (uint32_t)i * bytes
                              : high + ((uint32_t)i - nlow) * bytes;
  }
};

__device__ __forceinline__ Layout make_layout(uint32_t s0, uint32_t dyn_bytes,
                                              int want, uint32_t st, int32_t E) {
  Layout L;
  const uint32_t end = s0 + dyn_bytes;
  const uint32_t meta_bytes = 20u * (uint32_t)want + 16u + 4u * (uint32_t)(E + 1);
  L.meta = (end - meta_bytes) & ~15u;
  L.lut = (s0 + 0xFFFFu) & ~0xFFFFu;
  L.low = (s0 + 127u) & ~127u;
  L.nlow = L.low + st <= L.lut ? (L.lut - L.low) / st : 0u;
  L.high = L.lut + 65536u;
  const uint32_t nhigh = L.high + st <= L.meta ? (L.meta - L.high) / st : 0u;
  L.ns = (int)min((uint32_t)want, L.nlow + nhigh);
  if (L.high > L.meta) L.ns = 0;  // no room: the kernel reports and returns
  return L;
}

// Bounded wait until *flag == want (a value another thread of the block
// publishes); gives up like mbar_wait.
__device__ __forceinline__ bool flag_wait(const volatile int32_t* flag, int32_t want,
                                          volatile int* abort, int* err) {
  if (*flag == want) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 0;; ++it) {
    if (*flag == want) return true;
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

template <Fmt F, int G, int UPL>
__global__ void __launch_bounds__(kThreads, 1)
gemv_kernel(const GroupedProblem pb, const GemvPlan pl) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  uint32_t dyn_bytes;
  asm("mov.u32 %0, %%dynamic_smem_size;" : "=r"(dyn_bytes));
  const Layout lay = make_layout(smem_u32(smem_raw), dyn_bytes, pl.nstages,
                                 (uint32_t)pl.stage_bytes, pb.E);
  // generic pointers into the block's shared window
  uint8_t* const base = smem_raw - smem_u32(smem_raw);
  uint64_t* full = reinterpret_cast<uint64_t*>(base + lay.meta);
  uint64_t* empty = full + pl.nstages;
  volatile int* abort = reinterpret_cast<volatile int*>(empty + pl.nstages);
  volatile int32_t* slot_blk = reinterpret_cast<volatile int32_t*>(empty + pl.nstages) + 4;
  int32_t* off_s = const_cast<int32_t*>(slot_blk) + pl.nstages;

  constexpr int RG = 32 / G;                // rows per warp-wide row group
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t K = pb.K, N = pb.N;
  const int64_t U = K / 32;                 // 16-byte units per row
  const int64_t nbn = N / pl.R;             // blocks per routed row
  const int64_t b0 = pl.nblocks * blockIdx.x / gridDim.x;
  const int64_t b1 = pl.nblocks * (blockIdx.x + 1) / gridDim.x;
  const int nmine = (int)(b1 - b0);
  const int NS = lay.ns;
  const int tpb = pl.R / (2 * RG);          // tasks (two row groups) per block
  if (NS < 1) {
    if (threadIdx.x == 0) raise_error(pb.err, GBW_DEVERR_TIMEOUT);
    return;
  }
  const int64_t srow = (F == Fmt::NF4) ? (K / 64) * 4 : K / 32;  // scale bytes per row

  if (threadIdx.x == 0) {
    for (int i = 0; i < NS; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], (uint32_t)tpb);
      slot_blk[i] = -1;
    }
    *abort = 0;
    fence_barrier_init();
  }
  // pair table: entry b -> bf16 (value of the even element, value of the odd
  // element) in every lane's column; 16-byte stores fill four columns
  for (int i = threadIdx.x; i < 256 * 8; i += kThreads) {
    const uint32_t b = (uint32_t)i >> 3;
    const uint32_t qe = (F == Fmt::NF4) ? (b >> 4) : (b & 15u);
    const uint32_t qo = (F == Fmt::NF4) ? (b & 15u) : (b >> 4);
    const uint32_t v =
        (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(code_value(F, qe))) |
        ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(code_value(F, qo))) << 16);
    *reinterpret_cast<uint4*>(base + lay.lut + b * 256 + (i & 7) * 16) = make_uint4(v, v, v, v);
  }
  load_offsets_clamped(pb.offsets, pb.E, pb.P, off_s, pb.err);  // barrier inside

  if (warp == 0) {
    // ---------------- producer: bulk copies of whole row blocks ----------
    // Blocks are issued in rounds of Z = min(32, NS): lane l issues block
    // round * Z + l.  Its slot was last used by the block NS earlier, which
    // belongs to an earlier round, so no lane ever waits on a sibling lane;
    // when the CTA's blocks fit the ring (the decode shapes) every copy is
    // issued in the first round.  After issuing, the lane publishes the
    // block id in the slot: a consumer waits for it before waiting on the
    // slot's phase, so no parity wait ever runs two phases ahead.
    const int Z = NS < 32 ? NS : 32;
    const uint32_t cbytes = (uint32_t)(pl.R * (K / 2));
    const uint32_t sbytes = pl.scales_staged ? (uint32_t)(pl.R * srow) : 0u;
    int issued = 0;  // blocks issued by this lane
    bool ok = true;
    for (int r0 = 0; r0 < nmine && ok; r0 += Z) {
      const int j = r0 + lane;
      const bool mine = lane < Z && j < nmine;
      bool good = true;
      if (mine) {
        const int s = j % NS;
        good = mbar_wait(&empty[s], ((uint32_t)(j / NS) & 1u) ^ 1u, abort, pb.err);
        if (good) {
          const int64_t b = b0 + j;
          const int32_t p = (int32_t)(b / nbn);
          const int64_t n0 = (b - (int64_t)p * nbn) * pl.R;
          const int64_t row = (int64_t)expert_of_row(off_s, pb.E, p) * N + n0;
          uint8_t* dst = base + lay.slot(s, (uint32_t)pl.stage_bytes);
          mbar_arrive_expect_tx(&full[s], cbytes + sbytes);
          bulk_load(dst, pb.w + row * (K / 2), cbytes, &full[s]);
          if (sbytes)
            bulk_load(dst + pl.scale_off,
                      reinterpret_cast<const uint8_t*>(pb.scale) + row * srow, sbytes, &full[s]);
          __threadfence_block();
          slot_blk[s] = j;
          ++issued;
        }
      }
      ok = __all_sync(0xffffffffu, good);
    }
    if (!ok) {
      // Copies still in flight must land before the CTA exits.  Only the
      // last NS blocks issued by the warp can be in flight (issuing block j
      // needed block j - NS consumed), and their slots were not reused, so
      // each lane drains its own blocks among them.
      const int last = issued > 0 ? (issued - 1) * Z + lane : -1;
      const int glast = __reduce_max_sync(0xffffffffu, last);
      for (int j = last; j >= 0 && j > glast - NS; j -= Z)
        mbar_drain(&full[j % NS], (uint32_t)(j / NS) & 1u);
    }
  } else {
    // ---------------- consumers ----------------
    // A task is two row groups of one block (2 * RG rows), computed
    // interleaved; tasks t = c, c + W, ... go to consumer warp c.
    const int c = warp - 1;
    const int li = lane % G, rs = lane / G;
    const uint32_t lut_lane = lay.lut | ((uint32_t)lane * 4u);
    const int ntasks = nmine * tpb;
    uint32_t xr[UPL][16];
    int64_t xkey = -1;                      // (token, pass) the x registers hold
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
      xkey = (int64_t)tok * pl.npass + pass;
    };
    auto scale_of = [&](uint32_t st, int r, int64_t u, int32_t p, int64_t n0) -> float {
      if (F == Fmt::NF4) {
        return pl.scales_staged
                   ? __uint_as_float(lds32(st + pl.scale_off + (uint32_t)(r * srow + (u >> 1) * 4)))
                   : __ldg(reinterpret_cast<const float*>(pb.scale) +
                           ((int64_t)expert_of_row(off_s, pb.E, p) * N + n0 + r) * (K / 64) + (u >> 1));
      }
      uint32_t sb;
      if (pl.scales_staged) {
        const uint32_t a = st + pl.scale_off + (uint32_t)(r * srow + u);
        sb = (lds32(a & ~3u) >> ((a & 3u) * 8)) & 0xFFu;
      } else {
        sb = __ldg(reinterpret_cast<const uint8_t*>(pb.scale) +
                   ((int64_t)expert_of_row(off_s, pb.E, p) * N + n0 + r) * (K / 32) + u);
      }
      return e8m0_f32(sb);
    };
    // Block state of task t (block j = t / tpb) advanced by carry: a runtime
    // 64-bit division per task is a long dependent chain.
    int t = c;
    int j = t / tpb, sub = t - j * tpb;
    int s = j % NS;
    uint32_t ph = (uint32_t)(j / NS) & 1u;
    int64_t nbi = (b0 + j) % nbn;
    int32_t p = (int32_t)((b0 + j) / nbn);
    int32_t tok = t < ntasks ? token_of_row(pb.row_to_token, p, pb.T, pb.err) : 0;
    // The activations of the first task do not depend on the staged
    // weights: load them while its copy is in flight.
    if (t < ntasks) load_x(tok, 0);
    while (t < ntasks) {
      if (!__all_sync(0xffffffffu, flag_wait(&slot_blk[s], j, abort, pb.err) &&
                                       mbar_wait(&full[s], ph, abort, pb.err)))
        break;
      const int64_t n0 = nbi * pl.R;
      const uint32_t st = lay.slot(s, (uint32_t)pl.stage_bytes);
      const int ra = (2 * sub) * RG + rs, rb = ra + RG;  // rows of the two groups
      float ta = 0.0f, tb = 0.0f;
      for (int pass = 0; pass < pl.npass; ++pass) {
        if ((int64_t)tok * pl.npass + pass != xkey) load_x(tok, pass);
#pragma unroll
        for (int i = 0; i < UPL; ++i) {
          const int64_t u = ((int64_t)pass * UPL + i) * G + li;
          if (u < U) {
            const uint4 qa = lds128(st + (uint32_t)(ra * (K / 2) + u * 16));
            const uint4 qb = lds128(st + (uint32_t)(rb * (K / 2) + u * 16));
            const float sa = scale_of(st, ra, u, p, n0), sb = scale_of(st, rb, u, p, n0);
            ta = fmaf(dot_unit(qa, xr[i], lut_lane), sa, ta);
            tb = fmaf(dot_unit(qb, xr[i], lut_lane), sb, tb);
          }
        }
      }
      // Reduce both rows over the G lanes at once: the lower half of the
      // lanes collects row a, the upper half row b, then each half reduces.
      const bool hi = (li & (G / 2)) != 0;
      float keep = hi ? tb : ta;
      keep += __shfl_xor_sync(0xffffffffu, hi ? ta : tb, G / 2, G);
#pragma unroll
      for (int o = G / 4; o; o >>= 1) keep += __shfl_xor_sync(0xffffffffu, keep, o, G);
      if ((li & (G / 2 - 1)) == 0)
        pb.out[(int64_t)p * N + n0 + (hi ? rb : ra)] =
            __bfloat16_as_ushort(__float2bfloat16_rn(keep));
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
      // next task: t + W, moving the block state forward block by block
      t += kConsumers;
      sub += kConsumers;
      bool moved = false;
      while (sub >= tpb && j + 1 < nmine) {
        sub -= tpb;
        ++j;
        if (++s == NS) { s = 0; ph ^= 1u; }
        if (++nbi == nbn) { nbi = 0; ++p; moved = true; }
      }
      if (moved && t < ntasks) tok = token_of_row(pb.row_to_token, p, pb.T, pb.err);
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

template <Fmt F, int G, int UPL>
cudaError_t launch_t(const GroupedProblem& pb, const GemvPlan& pl, int grid,
                     cudaStream_t s) {
  auto k = gemv_kernel<F, G, UPL>;
  const size_t smem = kSmemCap;  // the kernel lays out the whole window
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  k<<<grid, kThreads, smem, s>>>(pb, pl);
  return cudaGetLastError();
}

template <Fmt F>
cudaError_t launch_f(const GroupedProblem& pb, const Shape& sh, const GemvPlan& pl,
                     int grid, cudaStream_t s) {
#define GBW_GEMV_CASE(GG, UU) \
  if (sh.G == GG && sh.UPL == UU) return launch_t<F, GG, UU>(pb, pl, grid, s);
  GBW_GEMV_CASE(32, 1) GBW_GEMV_CASE(32, 2) GBW_GEMV_CASE(32, 3)
  GBW_GEMV_CASE(16, 1) GBW_GEMV_CASE(16, 2) GBW_GEMV_CASE(16, 3)
  GBW_GEMV_CASE(8, 1) GBW_GEMV_CASE(8, 2) GBW_GEMV_CASE(8, 3)
  GBW_GEMV_CASE(4, 1) GBW_GEMV_CASE(4, 2) GBW_GEMV_CASE(4, 3)
#undef GBW_GEMV_CASE
  return cudaErrorInvalidValue;
}

}  // namespace

// Plans the GEMV for this problem; false when no ring of two slots fits in
// shared memory (rows too long).
bool gemv_plan(Fmt f, const GroupedProblem& pb, int num_sms, GemvPlan* out,
               Shape* shape, int* grid) {
  const int64_t K = pb.K;
  const Shape sh = pick_shape(K / 32);
  const int RG = 32 / sh.G;
  const int64_t srow = (f == Fmt::NF4) ? (K / 64) * 4 : K / 32;
  // the window holds the table, two partial slot regions around it (one
  // slot of each may be lost to fragmentation) and the barriers / offsets
  const int64_t fixed = 1024 + kLutBytes + 16 + 4 * (int64_t)(pb.E + 1);
  for (int R : {8, 4, 2, 1}) {
    if (R % (2 * RG) || pb.N % R) continue;  // whole tasks of two row groups
    GemvPlan pl{};
    pl.R = R;
    pl.npass = sh.npass;
    pl.nblocks = pb.P * (pb.N / R);
    const int64_t cbytes = (int64_t)R * (K / 2);
    const int64_t sbytes = (int64_t)R * srow;
    const uintptr_t sbase = reinterpret_cast<uintptr_t>(pb.scale);
    // a block's scales start at (e*N + n0) * srow: 16-byte aligned for every
    // block when the base, R * srow and the per-row step allow it
    pl.scales_staged = (sbase % 16 == 0) && (sbytes % 16 == 0) ? 1 : 0;
    pl.scale_off = (int32_t)cbytes;
    int64_t st = cbytes + (pl.scales_staged ? sbytes : 0);
    st = (st + 127) & ~int64_t(127);
    pl.stage_bytes = (int32_t)st;
    const int g = (int)std::min<int64_t>(num_sms, pl.nblocks);
    const int64_t per_cta = (pl.nblocks + g - 1) / g;
    const int64_t room = ((int64_t)kSmemCap - fixed) / (st + 16) - 2;
    if (room < 2) continue;
    pl.nstages = (int32_t)std::max<int64_t>(1, std::min<int64_t>(room, per_cta));
    *out = pl;
    *shape = sh;
    *grid = g;
    return true;
  }
  return false;
}

bool gemv_fits(Fmt f, const GroupedProblem& pb, int num_sms) {
  GemvPlan pl;
  Shape sh;
  int grid = 0;
  return pb.P == 0 || gemv_plan(f, pb, num_sms, &pl, &sh, &grid);
}

cudaError_t launch_gemv(Fmt f, const GroupedProblem& pb, int num_sms,
                        cudaStream_t s) {
  if (pb.P == 0 || pb.N == 0) return cudaSuccess;
  GemvPlan pl;
  Shape sh;
  int grid = 0;
  if (!gemv_plan(f, pb, num_sms, &pl, &sh, &grid)) return cudaErrorInvalidValue;
  return f == Fmt::NF4 ? launch_f<Fmt::NF4>(pb, sh, pl, grid, s)
                       : launch_f<Fmt::MXFP4>(pb, sh, pl, grid, s);
}

}  // namespace gbw
