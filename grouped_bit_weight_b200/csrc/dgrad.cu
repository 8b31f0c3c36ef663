// dgrad.cu -- grouped 4-bit activation gradient dx = dy * W on tcgen05
// (NF4 and MXFP4).
//
// "grouped-nf4-gemm 0.43.0", "Which entry point?": dgrad_4bit_grouped;
// "Receipts-driven engineering": the NF4 path is differentiable and
// fine-tuning never leaves the packed format.  For out = x W^T per expert,
//   dx[p, k] = sum_n dy[p, n] * W_e(p)[n, k].
// The reduction now runs over the weight rows n, and the scale blocks lie
// along the output dimension k, so the weights are read packed in the
// transposed orientation.
//
// B200 design (one persistent CTA per SM, 16 warps):
//   tile = up to 256 routed rows x 256 output columns k (MMA N), reduced
//          over N in stages of 64 weight rows; the routed rows go 128 at a
//          time (MMA M) to the two TMEM accumulator halves, both fed by one
//          decoded B stage, so a weight slab is decoded once per 256 rows;
//   warp 0      TMA: dy tile [256 x 64] (128B swizzle, K-major A operand)
//               and the packed slab [64 weight rows x 128 bytes] (swizzled so
//               the decode reads are bank-conflict free) -> smem ring (3)
//   warps 4-11  decode: thread (weight row n, 64-wide k block j) decodes 64
//               weights with the register table and stores them as one
//               128-byte row of the MN-major, 128B-swizzled B operand
//               (3-stage ring); the decoded tile lives only in smem
//   warp 1      tcgen05.mma (A and B from smem, fp32 accumulator in TMEM)
//   warps 12-15 epilogue: tcgen05.ld -> bf16 -> 16-byte stores of dx rows.
//               Tiles of up to 128 rows alternate between the two TMEM
//               accumulator halves (2 x 256 columns), so the epilogue of one
//               overlaps the mainloop of the next; a wider tile takes both.
// Tiles (expert, k tile, routed-row tile) with routed-row tiles innermost, so
// CTAs running together share one packed weight slab through L2.
#include "common.cuh"
#include "decode.cuh"

namespace gbw {
namespace {

constexpr int BM = 128;   // routed rows per accumulator half (MMA M)
constexpr int BMW = 256;  // routed rows per tile: two halves share each decoded B
constexpr int BN = 256;   // output k columns per tile (MMA N)
constexpr int BR = 64;    // weight rows (reduction) per stage
constexpr int LS = 3;     // load ring stages (dy + packed)
constexpr int DS = 3;     // decoded-B ring stages
constexpr int kThreads = 512;
constexpr uint32_t kTmemCols = 512;
static_assert(BR == 64, "the MMA issuer unrolls four 16-row steps per stage");

constexpr int kAStageBytes = BMW * BR * 2;  // 32 KB
constexpr int kAHalfBytes = BM * BR * 2;    // 16 KB
constexpr int kWStageBytes = BR * BN / 2;   // 8 KB
constexpr int kLStageBytes = kAStageBytes + kWStageBytes;
constexpr int kBStageBytes = BR * BN * 2;   // 32 KB

struct Smem {
  static constexpr int ld = 0;
  static constexpr int b = ld + LS * kLStageBytes;
  static constexpr int bars = b + DS * kBStageBytes;
  static constexpr int nbars = 2 * LS + 2 * DS + 4 + 1;
  static constexpr int misc = bars + nbars * 8;
  static constexpr int tables = misc + 16;
};

struct DTile {
  int32_t e, k0, p0, nv;
};

__device__ __forceinline__ DTile dtile_info(int64_t t, const int32_t* off,
                                            const int32_t* ts, int32_t E) {
  int32_t lo = 0, hi = E - 1;
  while (lo < hi) {
    int32_t mid = (lo + hi + 1) >> 1;
    if (ts[mid] <= t) lo = mid; else hi = mid - 1;
  }
  const int32_t cnt = off[lo + 1] - off[lo];
  const int32_t mt_n = (cnt + BMW - 1) / BMW;
  const int32_t u = (int32_t)(t - ts[lo]);
  const int32_t kt = u / mt_n, mt = u - kt * mt_n;
  DTile d;
  d.e = lo;
  d.k0 = kt * BN;
  d.p0 = off[lo] + mt * BMW;
  d.nv = min(BMW, cnt - mt * BMW);
  return d;
}

// Which accumulator half (256 TMEM columns) a tile uses: a tile of up to
// 128 routed rows takes the next half and the halves alternate, so its
// epilogue overlaps the next tile's mainloop; a wider tile takes both (the
// next one first).  The MMA thread and the epilogue warps step identical
// copies, so they agree on halves and on each half's barrier phase.
struct AccSched {
  uint32_t h = 0;
  uint32_t use0 = 0, use1 = 0;
  __device__ __forceinline__ uint32_t phase(uint32_t k) const { return (k ? use1 : use0) & 1u; }
  __device__ __forceinline__ void next(bool wide) {
    if (wide) {
      ++use0;
      ++use1;
    } else {
      if (h) ++use1; else ++use0;
      h ^= 1u;
    }
  }
};

template <Fmt F>
__global__ void __launch_bounds__(kThreads, 1)
dgrad_kernel(const GroupedProblem pb, const __grid_constant__ CUtensorMap tma,
             const __grid_constant__ CUtensorMap tmw) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Smem::bars);
  uint64_t* ld_full = bars;
  uint64_t* ld_empty = ld_full + LS;
  uint64_t* b_full = ld_empty + LS;
  uint64_t* b_empty = b_full + DS;
  uint64_t* acc_full = b_empty + DS;   // [2]
  uint64_t* acc_empty = acc_full + 2;  // [2]
  uint64_t* mma_done = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Smem::misc);
  volatile int* abort = reinterpret_cast<volatile int*>(smem + Smem::misc + 4);
  int32_t* off_s = reinterpret_cast<int32_t*>(smem + Smem::tables);
  int32_t* ts_s = off_s + (pb.E + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int32_t E = pb.E;
  const int64_t N = pb.N;  // reduction length (weight rows)
  const int64_t K = pb.K;  // output width
  const int NS = (int)(N / BR);
  const int32_t nkt = (int32_t)((K + BN - 1) / BN);

  if (threadIdx.x == 0) {
    for (int i = 0; i < LS; ++i) { mbar_init(&ld_full[i], 1); mbar_init(&ld_empty[i], 1 + 8); }
    for (int i = 0; i < DS; ++i) { mbar_init(&b_full[i], 8); mbar_init(&b_empty[i], 1); }
    for (int i = 0; i < 2; ++i) { mbar_init(&acc_full[i], 1); mbar_init(&acc_empty[i], 4); }
    mbar_init(mma_done, 1);
    *abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tma);
    tma_prefetch_desc(&tmw);
  }
  load_offsets_clamped(pb.offsets, E, pb.P, off_s, pb.err);
  tile_prefix(off_s, E, BMW, nkt, ts_s);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int64_t ntiles = ts_s[E];

  if (warp == 0) {
    // ---------------- loads: dy tile + packed slab ----------------
    if (lane == 0) {
      uint32_t g = 0;
      bool ok = true;
      for (int64_t t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
        const DTile d = dtile_info(t, off_s, ts_s, E);
        for (int ks = 0; ks < NS; ++ks, ++g) {
          const uint32_t s = g % LS, ph = (g / LS) & 1u;
          if (!(ok = mbar_wait(&ld_empty[s], ph ^ 1u, abort, pb.err))) break;
          uint8_t* st = smem + Smem::ld + s * kLStageBytes;
          mbar_arrive_expect_tx(&ld_full[s], kLStageBytes);
          tma_load_2d(st, &tma, ks * BR, d.p0, &ld_full[s]);
          tma_load_2d(st + kAStageBytes, &tmw, d.k0 / 2,
                      (int32_t)((int64_t)d.e * N + (int64_t)ks * BR), &ld_full[s]);
        }
      }
      if (*abort)
        for (uint32_t i = (g > LS ? g - LS : 0); i < g; ++i)
          mbar_drain(&ld_full[i % LS], (i / LS) & 1u);
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      uint32_t g = 0;
      bool ok = true;
      // descriptors advance by 64-bit adds (start address in 16-byte units):
      // nothing but the MMAs runs between them in this thread
      const uint64_t adesc0 = make_sdesc_sw128(smem_u32(smem + Smem::ld), 16, 1024);
      const uint64_t bdesc0 = make_sdesc_sw128(smem_u32(smem + Smem::b), 1024, 4096);
      AccSched acc;
      for (int64_t t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
        const DTile d = dtile_info(t, off_s, ts_s, E);
        const bool wide = d.nv > BM;
        const uint32_t nmma = (uint32_t)min((int64_t)BN, K - d.k0);
        const uint32_t idesc = make_idesc_bf16(BM, nmma, 0, 1);
        const uint32_t h0 = acc.h, h1 = acc.h ^ 1u;
        if (!(ok = mbar_wait(&acc_empty[h0], acc.phase(h0) ^ 1u, abort, pb.err))) break;
        if (wide && !(ok = mbar_wait(&acc_empty[h1], acc.phase(h1) ^ 1u, abort, pb.err))) break;
        tc_fence_after();
        const uint32_t d0 = tmem + h0 * 256u, d1 = tmem + h1 * 256u;
        for (int ks = 0; ks < NS; ++ks, ++g) {
          const uint32_t ls = g % LS, bs = g % DS;
          if (!(ok = mbar_wait(&ld_full[ls], (g / LS) & 1u, abort, pb.err))) break;
          if (!(ok = mbar_wait(&b_full[bs], (g / DS) & 1u, abort, pb.err))) break;
          tc_fence_after();
          const uint64_t ad = adesc0 + (uint64_t)((ls * kLStageBytes) >> 4);
          const uint64_t bd = bdesc0 + (uint64_t)((bs * kBStageBytes) >> 4);
          // one decoded B stage feeds both halves of a wide tile
          tc_mma_ss(d0, ad, bd, idesc, ks != 0);
          tc_mma_ss(d0, ad + 2, bd + 512, idesc, 1u);   // A +32 B, B +8 KB: next 16 n
          tc_mma_ss(d0, ad + 4, bd + 1024, idesc, 1u);
          tc_mma_ss(d0, ad + 6, bd + 1536, idesc, 1u);
          if (wide) {
            const uint64_t ad1 = ad + (uint64_t)(kAHalfBytes >> 4);  // dy rows 128..255
            tc_mma_ss(d1, ad1, bd, idesc, ks != 0);
            tc_mma_ss(d1, ad1 + 2, bd + 512, idesc, 1u);
            tc_mma_ss(d1, ad1 + 4, bd + 1024, idesc, 1u);
            tc_mma_ss(d1, ad1 + 6, bd + 1536, idesc, 1u);
          }
          tc_commit(&ld_empty[ls]);
          tc_commit(&b_empty[bs]);
        }
        if (!ok) break;
        tc_commit(&acc_full[h0]);
        if (wide) tc_commit(&acc_full[h1]);
        acc.next(wide);
      }
      tc_commit(mma_done);
      mbar_drain(mma_done, 0);
    }
  } else if (warp >= 4 && warp < 12) {
    // ---------------- decode into the MN-major B operand ----------------
    const int dw = warp - 4;
    const int j = dw >> 1;                      // 64-wide k block of the tile
    const int n = ((dw & 1) << 5) | lane;       // weight row within the stage
    const int rr = n & 7;                       // row inside the 8-row atom
    const int64_t my_tiles = blockIdx.x < ntiles ? (ntiles - 1 - blockIdx.x) / gridDim.x + 1 : 0;
    const uint32_t total = (uint32_t)(my_tiles * NS);
    // These warps bound the kernel by the instructions they issue, so the
    // bookkeeping is incremental: a cursor (local tile, stage) per
    // look-ahead distance steps one stage at a time and looks a tile up only
    // when it enters a new one (no divisions by the stage count), and the
    // scales of stage g + 4 are loaded into the slot stage g has just used
    // (fixed slots: a queue rotated by register copies would wait on each
    // load one stage after issuing it).
    struct Cursor {
      int64_t tl;
      int ks;
    };
    // scale cursor: the scales of (weight row n, block j) in its tile -- NF4
    // one fp32 absmax per 64-k block, MXFP4 two e8m0 bytes (two 32-blocks)
    Cursor sc_cur{0, 0};
    constexpr int kSB = F == Fmt::NF4 ? 4 : 2;           // scale bytes per 64-k block
    const int64_t srow_bytes = F == Fmt::NF4 ? (K / 64) * 4 : K / 32;
    const uint8_t* srow = nullptr;  // scales of weight row (e*N + n) at block j, or null
    auto srow_of = [&](int64_t tl) -> const uint8_t* {
      const DTile d = dtile_info(blockIdx.x + tl * gridDim.x, off_s, ts_s, E);
      if (d.k0 + 64 * j >= K) return nullptr;
      return reinterpret_cast<const uint8_t*>(pb.scale) + ((int64_t)d.e * N + n) * srow_bytes +
             (int64_t)(d.k0 / 64 + j) * kSB;
    };
    uint32_t sc_g = 0;  // stage the scale cursor points at
    if (total) srow = srow_of(0);
    auto scale_next = [&]() -> uint32_t {
      uint32_t v = 0u;
      if (sc_g < total) {
        if (srow) {
          const uint8_t* a = srow + (int64_t)sc_cur.ks * BR * srow_bytes;
          v = F == Fmt::NF4 ? __ldg(reinterpret_cast<const uint32_t*>(a))
                            : (uint32_t)__ldg(reinterpret_cast<const uint16_t*>(a));
        }
        ++sc_g;
        if (++sc_cur.ks == NS) {
          sc_cur.ks = 0;
          ++sc_cur.tl;
          if (sc_g < total) srow = srow_of(sc_cur.tl);
        }
      }
      return v;
    };
    uint32_t sA = scale_next(), sB = scale_next(), sC = scale_next(), sD = scale_next();
    Cursor cur{0, 0};
    bool jvalid = total ? dtile_info(blockIdx.x, off_s, ts_s, E).k0 + 64 * j < K : false;
    uint32_t ls = 0, lph = 0, bs = 0, bph = 0;  // ring slots and parities of stage g
    auto stage = [&](uint32_t sv) -> bool {
      if (!__all_sync(0xffffffffu, mbar_wait(&ld_full[ls], lph, abort, pb.err))) return false;
      // packed slab row n, bytes 32j .. 32j+31, stored 128B-swizzled
      const uint8_t* wst = smem + Smem::ld + ls * kLStageBytes + kAStageBytes + n * 128;
      const uint4 q0 = *reinterpret_cast<const uint4*>(wst + (((2 * j) ^ rr) << 4));
      const uint4 q1 = *reinterpret_cast<const uint4*>(wst + (((2 * j + 1) ^ rr) << 4));
      uint32_t o[32];
      const uint32_t P[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
      if (F == Fmt::NF4) {
        const Planes tb = nf4_planes(__uint_as_float(sv));
#pragma unroll
        for (int i = 0; i < 8; ++i) decode_word<true>(P[i], tb, &o[4 * i]);
      } else {
        // two 32-blocks: bytes 0-15 (k 0..31) and 16-31 (k 32..63)
        const Planes t0 = mxfp4_planes(sv & 0xFFu);
#pragma unroll
        for (int i = 0; i < 4; ++i) decode_word<false>(P[i], t0, &o[4 * i]);
        const Planes t1 = mxfp4_planes((sv >> 8) & 0xFFu);
#pragma unroll
        for (int i = 4; i < 8; ++i) decode_word<false>(P[i], t1, &o[4 * i]);
      }
      // release the slab only once the decode has consumed what was loaded
      // from it: the refill is an async-proxy (TMA) write and must not
      // overtake shared-memory loads still in flight
      __syncwarp();
      if (lane == 0) mbar_arrive(&ld_empty[ls]);
      if (!__all_sync(0xffffffffu, mbar_wait(&b_empty[bs], bph ^ 1u, abort, pb.err))) return false;
      if (jvalid) {
        // K-row n of atom (n/8, j): 128 bytes, chunk c at (c ^ rr)
        uint8_t* dst = smem + Smem::b + bs * kBStageBytes + ((n >> 3) * 4 + j) * 1024 + rr * 128;
#pragma unroll
        for (int c = 0; c < 8; ++c)
          *reinterpret_cast<uint4*>(dst + ((c ^ rr) << 4)) =
              make_uint4(o[4 * c], o[4 * c + 1], o[4 * c + 2], o[4 * c + 3]);
      }
      // generic-proxy smem writes -> visible to the tensor core (async proxy)
      fence_proxy_async();
      __syncwarp();
      if (lane == 0) mbar_arrive(&b_full[bs]);
      // next stage
      if (++ls == LS) { ls = 0; lph ^= 1u; }
      if (++bs == DS) { bs = 0; bph ^= 1u; }
      if (++cur.ks == NS) {
        cur.ks = 0;
        ++cur.tl;
        if (cur.tl < my_tiles)
          jvalid = dtile_info(blockIdx.x + cur.tl * gridDim.x, off_s, ts_s, E).k0 + 64 * j < K;
      }
      return true;
    };
    for (uint32_t g = 0; g < total;) {
      if (!stage(sA)) break;
      sA = scale_next();
      if (++g >= total) break;
      if (!stage(sB)) break;
      sB = scale_next();
      if (++g >= total) break;
      if (!stage(sC)) break;
      sC = scale_next();
      if (++g >= total) break;
      if (!stage(sD)) break;
      sD = scale_next();
      ++g;
    }
  } else if (warp >= 12) {
    // ---------------- epilogue ----------------
    const uint32_t q = (uint32_t)warp & 3u;
    AccSched acc;
    bool ok = true;
    for (int64_t t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
      const DTile d = dtile_info(t, off_s, ts_s, E);
      const bool wide = d.nv > BM;
      for (int part = 0; part < (wide ? 2 : 1); ++part) {
      const uint32_t hf = part ? acc.h ^ 1u : acc.h;
      const int m = part * BM + (int)(q * 32 + lane);  // routed row in the tile
      ok = __all_sync(0xffffffffu, mbar_wait(&acc_full[hf], acc.phase(hf), abort, pb.err));
      if (!ok) break;
      tc_fence_after();
      const int width = (int)min((int64_t)BN, K - d.k0);
      const int nchunks = width >> 5;
      const uint32_t taddr = tmem + ((q * 32u) << 16) + hf * 256u;
      uint16_t* dst = pb.out + (int64_t)(d.p0 + m) * K + d.k0;
      for (int c = 0; c < nchunks; ++c) {
        uint32_t r[32];
        tmem_load_32x32b_x32(taddr + c * 32, r);
        if (c == nchunks - 1) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&acc_empty[hf]);
        }
        if (m < d.nv) {
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            uint4 o;
            o.x = pack_bf16x2(__uint_as_float(r[8 * v + 0]), __uint_as_float(r[8 * v + 1]));
            o.y = pack_bf16x2(__uint_as_float(r[8 * v + 2]), __uint_as_float(r[8 * v + 3]));
            o.z = pack_bf16x2(__uint_as_float(r[8 * v + 4]), __uint_as_float(r[8 * v + 5]));
            o.w = pack_bf16x2(__uint_as_float(r[8 * v + 6]), __uint_as_float(r[8 * v + 7]));
            reinterpret_cast<uint4*>(dst + c * 32)[v] = o;
          }
        }
      }
      }
      acc.next(wide);
    }
  }

  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace

cudaError_t make_map_2d(CUtensorMap* m, CUtensorMapDataType dt, const void* base,
                        uint64_t d0, uint64_t d1, uint64_t pitch, uint32_t b0,
                        uint32_t b1, CUtensorMapSwizzle sw);

cudaError_t launch_dgrad(Fmt f, const GroupedProblem& pb, int num_sms, cudaStream_t s) {
  if (pb.P == 0 || pb.K == 0) return cudaSuccess;
  CUtensorMap tma, tmw;
  // dy [P, N] bf16: box 64 (reduction) x 256 rows, 128B swizzle
  cudaError_t e = make_map_2d(&tma, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, pb.x,
                              (uint64_t)pb.N, (uint64_t)pb.P, (uint64_t)pb.N * 2,
                              BR, BMW, CU_TENSOR_MAP_SWIZZLE_128B);
  if (e != cudaSuccess) return e;
  // packed [E*N, K/2] u8: box 128 bytes x 64 rows, 128B swizzle
  e = make_map_2d(&tmw, CU_TENSOR_MAP_DATA_TYPE_UINT8, pb.w, (uint64_t)pb.K / 2,
                  (uint64_t)pb.E * (uint64_t)pb.N, (uint64_t)pb.K / 2, BN / 2, BR,
                  CU_TENSOR_MAP_SWIZZLE_128B);
  if (e != cudaSuccess) return e;
  static_assert(1024 + Smem::tables + 8 * (1024 + 1) <= 232448,
                "shared memory for 1024 experts exceeds the 227 KB a CTA can have");
  const size_t smem = 1024 + Smem::tables + sizeof(int32_t) * 2 * (size_t)(pb.E + 1);
  auto k = f == Fmt::NF4 ? dgrad_kernel<Fmt::NF4> : dgrad_kernel<Fmt::MXFP4>;
  e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  k<<<num_sms, kThreads, smem, s>>>(pb, tma, tmw);
  return cudaGetLastError();
}

}  // namespace gbw
