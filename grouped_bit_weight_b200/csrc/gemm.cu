// gemm.cu -- grouped 4-bit x bf16 matmul on the 5th-generation tensor cores.
//
// "grouped-nf4-gemm 0.43.0", opening lines, and "Receipts-driven
// engineering", opening paragraph: one launch multiplies the routed rows of
// every active expert by that expert's packed weights; the codebook is
// decoded in registers inside the mainloop, with no bf16 copy of the weights
// in HBM.
//
// B200 design (one persistent CTA per SM, 16 warps):
//   tile  = 128 weight rows (MMA M) x up to 256 routed rows (MMA N) x K,
//           i.e. the matmul runs as out^T = W x^T ("swap AB"), so an expert
//           with few routed rows gets a narrow MMA N instead of a padded M;
//   warp 0      TMA: packed weight tiles [128 rows x 32 B] -> smem ring (8)
//   warp 2      TMA tile::gather4: the tile's x rows (through row_to_token)
//               -> 128B-swizzled smem ring (4 stages of 64 K)
//   warps 4-11  decode: each thread owns one weight row; per 64-K stage it
//               reads its 32 packed bytes, builds the block's bf16 table and
//               decodes with byte permutes, then writes 64 bf16 straight into
//               tensor memory (tcgen05.st) as the MMA's A operand -- the
//               decoded weights never touch shared or global memory; two
//               groups of four warps take alternate stages
//   warp 1      one thread issues tcgen05.mma (A from TMEM, B from smem,
//               fp32 accumulator in TMEM) and tcgen05.commit
//   warps 12-15 epilogue: tcgen05.ld the 128 x N accumulator, round to bf16,
//               transpose through smem, 16-byte stores of out rows
// Tensor memory: columns [0,256) accumulator, [256,512) an 8-stage ring of
// decoded A tiles (128 lanes x 32 columns of bf16x2 each).
// Scheduler: tiles (expert, 128-row weight tile, 256-row token tile) with
// zero-row experts skipped, enumerated from expert_offsets by every CTA and
// dealt round-robin (token tiles innermost, so CTAs running at the same time
// share one weight tile through L2).
#include "common.cuh"
#include "decode.cuh"

namespace gbw {
namespace {

constexpr int BM = 128;   // weight rows per tile (MMA M)
constexpr int BT = 256;   // routed rows per tile (max MMA N)
constexpr int BK = 64;    // K per stage
constexpr int XS = 4;     // activation ring stages
constexpr int WS = 8;     // packed-weight ring stages == TMEM A ring stages
constexpr int kThreads = 512;
constexpr uint32_t kAccCols = 256;
constexpr uint32_t kACol0 = 256;
constexpr uint32_t kTmemCols = 512;

constexpr int kXStageBytes = BT * BK * 2;      // 32 KB
constexpr int kWStageBytes = BM * BK / 2;      // 4 KB
constexpr int kEpiRowBytes = 80;               // 64 B of data + 16 B pad
constexpr int kEpiWarpBytes = 32 * kEpiRowBytes;

struct Smem {
  // byte offsets inside the dynamic shared memory block
  static constexpr int x = 0;
  static constexpr int w = x + XS * kXStageBytes;
  static constexpr int epi = w + WS * kWStageBytes;
  static constexpr int bars = epi + 4 * kEpiWarpBytes;
  static constexpr int nbars = 2 * XS + 4 * WS + 3;
  static constexpr int misc = bars + nbars * 8;  // tmem base, abort flag
  static constexpr int tables = misc + 16;       // offsets[E+1], tile_start[E+1]
};

struct TileInfo {
  int32_t e, n0, p0, nv;  // expert, first weight row, first routed row, rows
};

__device__ __forceinline__ TileInfo tile_info(int64_t t, const int32_t* off,
                                              const int32_t* ts, int32_t E,
                                              int32_t ntn) {
  int32_t lo = 0, hi = E - 1;  // last e with ts[e] <= t
  while (lo < hi) {
    int32_t mid = (lo + hi + 1) >> 1;
    if (ts[mid] <= t) lo = mid; else hi = mid - 1;
  }
  const int32_t cnt = off[lo + 1] - off[lo];
  const int32_t tt = (cnt + BT - 1) / BT;
  const int32_t u = (int32_t)(t - ts[lo]);
  const int32_t nt = u / tt, mt = u - nt * tt;
  TileInfo ti;
  ti.e = lo;
  ti.n0 = nt * BM;
  ti.p0 = off[lo] + mt * BT;
  ti.nv = min(BT, cnt - mt * BT);
  (void)ntn;
  return ti;
}

template <Fmt F>
__global__ void __launch_bounds__(kThreads, 1)
gemm_kernel(const GroupedProblem pb, const __grid_constant__ CUtensorMap tmx,
            const __grid_constant__ CUtensorMap tmw) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // 1024-byte alignment for the 128B-swizzled activation tiles
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Smem::bars);
  uint64_t* x_full = bars;
  uint64_t* x_empty = x_full + XS;
  uint64_t* w_full = x_empty + XS;
  uint64_t* w_empty = w_full + WS;
  uint64_t* a_full = w_empty + WS;
  uint64_t* a_empty = a_full + WS;
  uint64_t* acc_full = a_empty + WS;
  uint64_t* acc_empty = acc_full + 1;
  uint64_t* mma_done = acc_empty + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Smem::misc);
  volatile int* abort = reinterpret_cast<volatile int*>(smem + Smem::misc + 4);
  int32_t* off_s = reinterpret_cast<int32_t*>(smem + Smem::tables);
  int32_t* ts_s = off_s + (pb.E + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int32_t E = pb.E;
  const int64_t K = pb.K, N = pb.N;
  const int NK = (int)(K / BK);
  const int32_t ntn = (int32_t)((N + BM - 1) / BM);

  if (threadIdx.x == 0) {
    for (int i = 0; i < XS; ++i) { mbar_init(&x_full[i], 1); mbar_init(&x_empty[i], 1); }
    for (int i = 0; i < WS; ++i) {
      mbar_init(&w_full[i], 1);
      mbar_init(&w_empty[i], 4);
      mbar_init(&a_full[i], 4);
      mbar_init(&a_empty[i], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, 4);
    mbar_init(mma_done, 1);
    *abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmx);
    tma_prefetch_desc(&tmw);
  }
  load_offsets_clamped(pb.offsets, E, pb.P, off_s, pb.err);  // has __syncthreads
  if (threadIdx.x == 0) {
    int32_t acc = 0;
    for (int32_t e = 0; e < E; ++e) {
      ts_s[e] = acc;
      const int32_t cnt = off_s[e + 1] - off_s[e];
      acc += ntn * ((cnt + BT - 1) / BT);
    }
    ts_s[E] = acc;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int64_t ntiles = ts_s[E];

  if (warp == 0) {
    // ---------------- packed-weight producer ----------------
    if (lane == 0) {
      uint32_t g = 0;
      bool ok = true;
      for (int64_t t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
        const TileInfo ti = tile_info(t, off_s, ts_s, E, ntn);
        const int32_t row0 = (int32_t)((int64_t)ti.e * N + ti.n0);
        for (int kb = 0; kb < NK; ++kb, ++g) {
          const uint32_t s = g % WS, ph = (g / WS) & 1u;
          if (!(ok = mbar_wait(&w_empty[s], ph ^ 1u, abort, pb.err))) break;
          mbar_arrive_expect_tx(&w_full[s], kWStageBytes);
          tma_load_2d(smem + Smem::w + s * kWStageBytes, &tmw, kb * (BK / 2), row0,
                      &w_full[s]);
        }
      }
      // after an abort, let the copies already issued land first
      if (*abort)
        for (uint32_t i = (g > WS ? g - WS : 0); i < g; ++i)
          mbar_drain(&w_full[i % WS], (i / WS) & 1u);
    }
  } else if (warp == 2) {
    // ---------------- activation producer (row gather) ----------------
    uint32_t g = 0;
    bool ok = true;
    for (int64_t t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
      const TileInfo ti = tile_info(t, off_s, ts_s, E, ntn);
      const int ngroups = (ti.nv + 3) >> 2;  // gather4 groups (<= 64)
      int32_t tok[2][4];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int gi = lane + 32 * h;
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          int32_t row = 4 * gi + r;
          row = row < ti.nv ? row : ti.nv - 1;  // pad with the last valid row
          tok[h][r] = gi < ngroups
                          ? token_of_row(pb.row_to_token, ti.p0 + row, pb.T, pb.err)
                          : 0;
        }
      }
      for (int kb = 0; kb < NK; ++kb, ++g) {
        const uint32_t s = g % XS, ph = (g / XS) & 1u;
        int good = 1;
        if (lane == 0) {
          good = mbar_wait(&x_empty[s], ph ^ 1u, abort, pb.err);
          if (good) mbar_arrive_expect_tx(&x_full[s], (uint32_t)ngroups * 512u);
        }
        good = __shfl_sync(0xffffffffu, good, 0);
        if (!good) { ok = false; break; }
        uint8_t* dst = smem + Smem::x + s * kXStageBytes;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int gi = lane + 32 * h;
          if (gi < ngroups)
            tma_gather4(dst + gi * 512, &tmx, kb * BK, tok[h][0], tok[h][1],
                        tok[h][2], tok[h][3], &x_full[s]);
        }
      }
    }
    if (lane == 0 && *abort)
      for (uint32_t i = (g > XS ? g - XS : 0); i < g; ++i)
        mbar_drain(&x_full[i % XS], (i / XS) & 1u);
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      uint32_t g = 0, it = 0;
      bool ok = true;
      const uint32_t xbase = smem_u32(smem + Smem::x);
      for (int64_t t = blockIdx.x; t < ntiles && ok; t += gridDim.x, ++it) {
        const TileInfo ti = tile_info(t, off_s, ts_s, E, ntn);
        const uint32_t nmma = (uint32_t)((ti.nv + 15) & ~15);
        const uint32_t idesc = make_idesc_bf16(BM, nmma, 0, 0);
        if (!(ok = mbar_wait(acc_empty, (it & 1u) ^ 1u, abort, pb.err))) break;
        tc_fence_after();
        for (int kb = 0; kb < NK; ++kb, ++g) {
          const uint32_t xs = g % XS, ws = g % WS;
          if (!(ok = mbar_wait(&a_full[ws], (g / WS) & 1u, abort, pb.err))) break;
          if (!(ok = mbar_wait(&x_full[xs], (g / XS) & 1u, abort, pb.err))) break;
          tc_fence_after();
#pragma unroll
          for (int j = 0; j < BK / 16; ++j) {
            const uint64_t bdesc =
                make_sdesc_sw128(xbase + xs * kXStageBytes + j * 32, 16, 1024);
            tc_mma_ts(tmem, tmem + kACol0 + ws * 32 + j * 8, bdesc, idesc,
                      (kb | j) != 0);
          }
          tc_commit(&x_empty[xs]);
          tc_commit(&a_empty[ws]);
        }
        if (ok) tc_commit(acc_full);
      }
      // every MMA this thread issued has finished before TMEM is released
      tc_commit(mma_done);
      mbar_drain(mma_done, 0);
    }
  } else if (warp >= 4 && warp < 12) {
    // ---------------- decode ----------------
    const uint32_t grp = (uint32_t)(warp - 4) >> 2;  // stage parity handled
    const uint32_t q = (uint32_t)warp & 3u;          // TMEM lane quarter
    const int m = (int)(q * 32 + lane);              // weight row in tile
    const uint32_t tlane = tmem + ((q * 32u) << 16);
    uint32_t g = 0;
    bool ok = true;
    for (int64_t t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
      const TileInfo ti = tile_info(t, off_s, ts_s, E, ntn);
      const bool rvalid = ti.n0 + m < N;
      const int64_t wrow = (int64_t)ti.e * N + ti.n0 + m;
      for (int kb = 0; kb < NK; ++kb, ++g) {
        if ((g & 1u) != grp) continue;
        const uint32_t ws = g % WS, ph = (g / WS) & 1u;
        // block scale(s) of this row and stage
        float a = 0.0f;
        uint32_t s01 = 0;
        if (rvalid) {
          if (F == Fmt::NF4)
            a = __ldg(reinterpret_cast<const float*>(pb.scale) + wrow * (K / 64) + kb);
          else
            s01 = __ldg(reinterpret_cast<const uint16_t*>(
                reinterpret_cast<const uint8_t*>(pb.scale) + wrow * (K / 32) + 2 * kb));
        }
        ok = __all_sync(0xffffffffu, mbar_wait(&w_full[ws], ph, abort, pb.err));
        if (!ok) break;
        const uint4* src = reinterpret_cast<const uint4*>(smem + Smem::w + ws * kWStageBytes + m * 32);
        const uint4 q0 = src[0], q1 = src[1];
        __syncwarp();
        if (lane == 0) mbar_arrive(&w_empty[ws]);
        const uint32_t P[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
        uint32_t o[32];
        if (F == Fmt::NF4) {
          const Planes tb = nf4_planes(a);
#pragma unroll
          for (int i = 0; i < 8; ++i) decode_word<true>(P[i], tb, &o[4 * i]);
        } else {
          const Planes t0 = mxfp4_planes(s01 & 0xFFu);
#pragma unroll
          for (int i = 0; i < 4; ++i) decode_word<false>(P[i], t0, &o[4 * i]);
          const Planes t1 = mxfp4_planes(s01 >> 8);
#pragma unroll
          for (int i = 4; i < 8; ++i) decode_word<false>(P[i], t1, &o[4 * i]);
        }
        ok = __all_sync(0xffffffffu, mbar_wait(&a_empty[ws], ph ^ 1u, abort, pb.err));
        if (!ok) break;
        tc_fence_after();
        tmem_st_32x32b_x32(tlane + kACol0 + ws * 32, o);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&a_full[ws]);
      }
    }
  } else if (warp >= 12) {
    // ---------------- epilogue ----------------
    const uint32_t q = (uint32_t)warp & 3u;
    const uint32_t tlane = tmem + ((q * 32u) << 16);
    uint8_t* stage = smem + Smem::epi + q * kEpiWarpBytes;
    uint32_t it = 0;
    for (int64_t t = blockIdx.x; t < ntiles; t += gridDim.x, ++it) {
      const TileInfo ti = tile_info(t, off_s, ts_s, E, ntn);
      const bool ok = __all_sync(0xffffffffu, mbar_wait(acc_full, it & 1u, abort, pb.err));
      if (!ok) break;
      tc_fence_after();
      const int nchunks = (ti.nv + 31) >> 5;
      const int ncol0 = ti.n0 + (int)q * 32;  // first output column of this warp
      for (int c = 0; c < nchunks; ++c) {
        uint32_t r[32];
        tmem_ld_32x32b_x32(tlane + c * 32, r);
        tmem_wait_ld();
        if (c == nchunks - 1) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(acc_empty);
        }
        // thread = output column ncol0+lane, r[j] = routed row c*32+j
#pragma unroll
        for (int j = 0; j < 32; ++j)
          *reinterpret_cast<uint16_t*>(stage + j * kEpiRowBytes + lane * 2) =
              __bfloat16_as_ushort(__float2bfloat16_rn(__uint_as_float(r[j])));
        __syncwarp();
        const int row = c * 32 + lane;  // routed row within the tile
        if (row < ti.nv) {
          uint16_t* dst = pb.out + (int64_t)(ti.p0 + row) * N + ncol0;
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            if (ncol0 + v * 8 < N)
              reinterpret_cast<uint4*>(dst)[v] =
                  *reinterpret_cast<const uint4*>(stage + lane * kEpiRowBytes + v * 16);
          }
        }
        __syncwarp();
      }
    }
  }

  // ---------------- teardown ----------------
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, kTmemCols);
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t,
                                  void*, const cuuint64_t*, const cuuint64_t*,
                                  const cuuint32_t*, const cuuint32_t*,
                                  CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

}  // namespace

EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    cudaDriverEntryPointQueryResult q;
    void* p = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault,
                                &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// 2-D tensor map: inner dimension d0 elements (contiguous), outer d1 rows
// with a row pitch of `pitch` bytes.
cudaError_t make_map_2d(CUtensorMap* m, CUtensorMapDataType dt, const void* base,
                        uint64_t d0, uint64_t d1, uint64_t pitch, uint32_t b0,
                        uint32_t b1, CUtensorMapSwizzle sw) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return cudaErrorNotSupported;
  const cuuint64_t dims[2] = {d0, d1};
  const cuuint64_t strides[1] = {pitch};
  const cuuint32_t box[2] = {b0, b1};
  const cuuint32_t es[2] = {1, 1};
  CUresult r = enc(m, dt, 2, const_cast<void*>(base), dims, strides, box, es,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

size_t gemm_smem_bytes(int32_t E) {
  return 1024 + Smem::tables + sizeof(int32_t) * 2 * (size_t)(E + 1);
}

cudaError_t launch_gemm(Fmt f, const GroupedProblem& pb, int num_sms,
                        cudaStream_t s) {
  if (pb.P == 0 || pb.N == 0) return cudaSuccess;
  CUtensorMap tmx, tmw;
  cudaError_t e = make_map_2d(&tmx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, pb.x,
                              (uint64_t)pb.K, (uint64_t)pb.T, (uint64_t)pb.K * 2,
                              BK, 1, CU_TENSOR_MAP_SWIZZLE_128B);
  if (e != cudaSuccess) return e;
  e = make_map_2d(&tmw, CU_TENSOR_MAP_DATA_TYPE_UINT8, pb.w, (uint64_t)pb.K / 2,
                  (uint64_t)pb.E * (uint64_t)pb.N, (uint64_t)pb.K / 2, BK / 2, BM,
                  CU_TENSOR_MAP_SWIZZLE_NONE);
  if (e != cudaSuccess) return e;
  const size_t smem = gemm_smem_bytes(pb.E);
  auto k = (f == Fmt::NF4) ? gemm_kernel<Fmt::NF4> : gemm_kernel<Fmt::MXFP4>;
  e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem);
  if (e != cudaSuccess) return e;
  k<<<num_sms, kThreads, smem, s>>>(pb, tmx, tmw);
  return cudaGetLastError();
}

}  // namespace gbw
