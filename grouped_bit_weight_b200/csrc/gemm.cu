// gemm.cu -- grouped 4-bit x bf16 matmul on the 5th-generation tensor cores.
//
// "grouped-nf4-gemm 0.43.0", opening lines, and "Receipts-driven
// engineering", opening paragraph: one launch multiplies the routed rows of
// every active expert by that expert's packed weights; the codebook is
// decoded in registers inside the mainloop, with no bf16 copy of the weights
// in HBM.
//
// B200 design (one persistent CTA per SM, 16 warps):
//   tile  = 128 weight rows (MMA M) x up to 512 routed rows x K: the matmul
//           runs as out^T = W x^T ("swap AB"), so an expert with few routed
//           rows gets a narrow MMA N instead of a padded M.  Rows past 256
//           go to the second accumulator half, fed by the same decoded A
//           stage, so a large expert's weights are decoded half as often
//           (wide tiles: identity rows only; gathered rows keep 256-row
//           tiles, whose cp.async gather cannot feed 64 KB stages);
//   warps 4-11  decode, two groups of four warps taking alternate 64-K
//               stages.  A stage's packed bytes (128 rows x 32 bytes) arrive
//               by TMA into the group's 2-slot ring; a tile's scales (128
//               consecutive rows of one expert, one contiguous range) arrive
//               by one bulk copy into a double buffer.  Each thread owns one
//               weight row: it builds the block's bf16 table, decodes with
//               byte permutes and stores the 64 bf16 as one 128-byte row of
//               the 128B-swizzled, K-major A tile (one slot per group).
//               These warps bound the kernel by the instructions they issue,
//               so their loop does no per-stage divisions or global loads;
//   warp 2      activations, identity rows: 2-D TMA boxes (64 K x 256 rows,
//               128B swizzle; 32-row boxes for a partial half) into a
//               2-stage ring of 64 KB stages;
//   warps 0,2,3 activations gathered through row_to_token: eight consecutive
//               lanes copy one row's 128 bytes of a stage with 16-byte
//               cp.async, so each warp instruction moves four whole rows
//               (4-stage ring of 32 KB stages);
//   warp 1      allocates TMEM; one thread issues tcgen05.mma (A and B from
//               shared memory, fp32 accumulator in TMEM) and tcgen05.commit;
//   warps 12-15 epilogue: tcgen05.ld 32 accumulator columns (routed rows) of
//               the warp's 32 weight rows, round to bf16, transpose 32 x 32
//               through shared memory and write whole 64-byte row segments.
// Tensor memory holds two 128 x 256 fp32 accumulator halves: tiles of up to
// 256 rows alternate between them, so the epilogue of one overlaps the
// mainloop of the next; a wider tile takes both.
// SwiGLU variant (the gate_up projection of the fused expert pass): a tile
// holds 64 gate rows and the matching 64 up rows (two TMA boxes), and each
// decode thread writes gate row j to A-tile row 32*(j/16) + j%16 and up row
// j sixteen rows further.  Gate and up of one output column then land in
// TMEM lanes l and l + 16 of one epilogue warp, which pairs them with one
// shuffle and writes h = bf16(silu(bf16 gate) * bf16 up) -- no cross-warp
// exchange, and the decoded rows of a quarter-warp stay consecutive (no
// bank conflicts on the swizzled A-tile stores).
// Scheduler: tiles (expert, 128-row weight tile, token tile) with
// zero-row experts skipped, enumerated from expert_offsets by every CTA and
// dealt round-robin (token tiles innermost, so CTAs running at the same time
// share one weight tile through L2).
#include "common.cuh"
#include "decode.cuh"

namespace gbw {
namespace {

constexpr int BM = 128;   // weight rows per tile (MMA M)
constexpr int BH = 256;   // routed rows per accumulator half (max MMA N)
constexpr int BK = 64;    // K per stage
constexpr int kXRingBytes = 128 * 1024;  // activation ring, either tile shape
constexpr int kXSMax = 4;                // most activation stages (barriers)
constexpr int AS = 2;     // decoded-weight (A operand) ring stages: one per decode group
static_assert(AS % 2 == 0, "the two decode groups own alternate A slots");
constexpr int WG = 2;     // packed-weight ring stages per decode group
constexpr int kThreads = 512;
constexpr uint32_t kTmemCols = 512;  // two 256-column accumulators
static_assert(BK == 64, "the MMA issuer unrolls four K = 16 steps per stage");

constexpr int kXHalfBytes = BH * BK * 2;       // 32 KB

// Tile shapes.  Wide (identity rows, activations by TMA): up to 512 routed
// rows, both accumulator halves fed by one decoded A stage, so a large
// expert's weights are decoded half as often; two 64 KB activation stages.
// Narrow (gathered rows): up to 256 routed rows, four 32 KB stages -- the
// cp.async gather cannot keep two 64 KB stages fed.
template <bool W>
struct TileCfg {
  static constexpr int BT = W ? 512 : 256;
  static constexpr int XS = W ? 2 : 4;
  static constexpr int kXStageBytes = BT * BK * 2;
  static_assert(XS * kXStageBytes == kXRingBytes && XS <= kXSMax, "ring");
};
constexpr int kAStageBytes = BM * BK * 2;      // 16 KB
constexpr int kWStageBytes = BM * BK / 2;      // 4 KB: 128 rows x 32 packed bytes
constexpr int kScaleBuf = 16 * 1024;           // one tile's scales (double buffered)
constexpr int kGatherThreads = 96;             // warps 0, 2, 3
constexpr int kEpiRowBytes = 64;               // one transposed row (read 4 lanes a row: no conflicts)
constexpr int kEpiWarpBytes = 32 * kEpiRowBytes;

struct Smem {
  // byte offsets inside the dynamic shared memory block (1024-aligned base)
  static constexpr int x = 0;
  static constexpr int a = x + kXRingBytes;
  static constexpr int w = a + AS * kAStageBytes;    // packed weights, 2 groups
  static constexpr int sc = w + 2 * WG * kWStageBytes;   // tile scales, 2 buffers
  static constexpr int epi = sc + 2 * kScaleBuf;         // epilogue transpose
  static constexpr int bars = epi + 4 * kEpiWarpBytes;
  static constexpr int nbars = 2 * kXSMax + 2 * AS + 4 * WG + 4 + 5;
  static constexpr int misc = bars + nbars * 8;      // tmem base, abort flag
  static constexpr int tables = misc + 16;           // offsets[E+1], tile_start[E+1]
};

// Which accumulator half (256 TMEM columns) a tile uses.  A tile of up to
// 256 rows takes the next half and the halves alternate, so its epilogue
// overlaps the next tile's mainloop; a wider tile takes both halves (the
// next one first).  The MMA thread and the epilogue warps step identical
// copies, so they agree on halves and on each half's barrier phase.
struct AccSched {
  uint32_t h = 0;              // next half
  uint32_t use0 = 0, use1 = 0;  // tiles that have used each half so far
  // parity of the current use of half k (registers, no indexed array)
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

struct TileInfo {
  int32_t e, n0, p0, nv;  // expert, first weight row, first routed row, rows
};

__device__ __forceinline__ TileInfo tile_info(int64_t t, const int32_t* off,
                                              const int32_t* ts, int32_t E, int32_t BT,
                                              int32_t NS = BM) {
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
  ti.n0 = nt * NS;
  ti.p0 = off[lo] + mt * BT;
  ti.nv = min(BT, cnt - mt * BT);
  return ti;
}

template <Fmt F, bool W, bool kGLU>
__global__ void __launch_bounds__(kThreads, 1)
gemm_kernel(const GroupedProblem pb, const __grid_constant__ CUtensorMap tmx,
            const __grid_constant__ CUtensorMap tmx32,
            const __grid_constant__ CUtensorMap tmw,
            const __grid_constant__ CUtensorMap tmw64, const int srow,
            const int tile_scales, const int32_t glu_i) {
  // kGLU: pb.N = 2 * glu_i weight rows per expert (gate rows, then up rows);
  // a tile covers NS = 64 gate columns; out is h [P, glu_i]
  constexpr int NS = kGLU ? 64 : BM;
  constexpr int BT = TileCfg<W>::BT;  // routed rows per tile
  constexpr int XS = TileCfg<W>::XS;  // activation ring stages
  constexpr int kXStageBytes = TileCfg<W>::kXStageBytes;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // 1024-byte alignment for the 128B-swizzled tiles
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Smem::bars);
  uint64_t* x_full = bars;
  uint64_t* x_empty = x_full + XS;
  uint64_t* a_full = x_empty + XS;
  uint64_t* a_empty = a_full + AS;
  uint64_t* w_full = a_empty + AS;     // [2][WG]
  uint64_t* w_empty = w_full + 2 * WG; // [2][WG]
  uint64_t* sc_full = w_empty + 2 * WG;  // [2]
  uint64_t* sc_empty = sc_full + 2;      // [2]
  uint64_t* acc_full = sc_empty + 2;     // [2]
  uint64_t* acc_empty = acc_full + 2;  // [2]
  uint64_t* mma_done = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Smem::misc);
  volatile int* abort = reinterpret_cast<volatile int*>(smem + Smem::misc + 4);
  int32_t* off_s = reinterpret_cast<int32_t*>(smem + Smem::tables);
  int32_t* ts_s = off_s + (pb.E + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int32_t E = pb.E;
  const int64_t K = pb.K, N = pb.N;
  // K % 64 == 32 (plain MXFP4 matmuls only; NF4 and the SwiGLU tiles need
  // K % 64 == 0): the last stage is half a stage.  Its upper 32 K are zeros
  // on both sides -- activations by the TMA's out-of-range fill or a
  // zero-filling gather copy, packed weights by the TMA's fill (code 0,
  // decoded with scale 2^0 to +0) -- so they add nothing to the sums.  The
  // other kernels compile without the tail code: the gather warps' loop
  // bounds the gathered path and is kept minimal.
  constexpr bool kTail = F == Fmt::MXFP4 && !kGLU;
  const int NK = kTail ? (int)((K + BK - 1) / BK) : (int)(K / BK);
  const int32_t ntn = kGLU ? glu_i / NS : (int32_t)((N + BM - 1) / BM);
  const int64_t ON = kGLU ? (int64_t)glu_i : N;  // columns of out
  const bool gathered = pb.row_to_token != nullptr;

  if (threadIdx.x == 0) {
    // TMA: one arrival plus bytes; gather: every gather thread arrives
    const uint32_t xcount = gathered ? (uint32_t)kGatherThreads : 1u;
    for (int i = 0; i < XS; ++i) { mbar_init(&x_full[i], xcount); mbar_init(&x_empty[i], 1); }
    for (int i = 0; i < AS; ++i) { mbar_init(&a_full[i], 4); mbar_init(&a_empty[i], 1); }
    for (int i = 0; i < 2 * WG; ++i) { mbar_init(&w_full[i], 1); mbar_init(&w_empty[i], 4); }
    for (int i = 0; i < 2; ++i) { mbar_init(&sc_full[i], 1); mbar_init(&sc_empty[i], 8); }
    for (int i = 0; i < 2; ++i) { mbar_init(&acc_full[i], 1); mbar_init(&acc_empty[i], 4); }
    mbar_init(mma_done, 1);
    *abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  if (warp == 2 && lane == 0 && !gathered) {
    tma_prefetch_desc(&tmx);
    tma_prefetch_desc(&tmx32);
  }
  if ((warp == 4 || warp == 8) && lane == 0) tma_prefetch_desc(kGLU ? &tmw64 : &tmw);
  load_offsets_clamped(pb.offsets, E, pb.P, off_s, pb.err);  // has __syncthreads
  tile_prefix(off_s, E, BT, ntn, ts_s);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int64_t ntiles = ts_s[E];

  if (warp == 0 || warp == 2 || warp == 3) {
    // ---------------- activation producer ----------------
    uint32_t g = 0;
    bool ok = true;
    if (!gathered) {
      // routed row p reads x row p: per stage, each 256-row half of the
      // tile is one 2-D TMA box (64 K x 256 rows), or only the 32-row boxes
      // a partial half uses (most experts end in a partial tile)
      if (warp == 2 && lane == 0) {
        for (int64_t t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
          const TileInfo ti = tile_info(t, off_s, ts_s, E, BT, NS);
          for (int kb = 0; kb < NK; ++kb, ++g) {
            const uint32_t s = g % XS, ph = (g / XS) & 1u;
            if (!(ok = mbar_wait(&x_empty[s], ph ^ 1u, abort, pb.err))) break;
            uint8_t* dst = smem + Smem::x + s * kXStageBytes;
            // each half: one 256-row box when full, else the 32-row boxes it uses
            const int n0 = min(ti.nv, BH), n1 = ti.nv - n0;
            const int b0 = n0 == BH ? 0 : (n0 + 31) >> 5;
            const int b1 = n1 == BH ? 0 : (n1 + 31) >> 5;
            const uint32_t bytes = (n0 == BH ? kXHalfBytes : b0 * (32 * BK * 2)) +
                                   (n1 == BH ? kXHalfBytes : b1 * (32 * BK * 2));
            mbar_arrive_expect_tx(&x_full[s], bytes);
            if (n0 == BH) tma_load_2d(dst, &tmx, kb * BK, ti.p0, &x_full[s]);
            for (int b = 0; b < b0; ++b)
              tma_load_2d(dst + b * (32 * BK * 2), &tmx32, kb * BK, ti.p0 + 32 * b, &x_full[s]);
            if (n1 == BH) tma_load_2d(dst + kXHalfBytes, &tmx, kb * BK, ti.p0 + BH, &x_full[s]);
            for (int b = 0; b < b1; ++b)
              tma_load_2d(dst + kXHalfBytes + b * (32 * BK * 2), &tmx32, kb * BK,
                          ti.p0 + BH + 32 * b, &x_full[s]);
          }
        }
        if (*abort)
          for (uint32_t i = (g > XS ? g - XS : 0); i < g; ++i)
            mbar_drain(&x_full[i % XS], (i / XS) & 1u);
      }
    } else {
      // Gathered rows.  Lane l of gather warp w copies 16-byte chunk (l & 7)
      // of rows 4w + (l >> 3) + 12i: eight lanes cover one row's 128 bytes,
      // so a warp instruction moves four whole rows.  Chunk c of row r lands
      // at (c ^ (r % 8)) -- the 128-byte swizzle the MMA's descriptor
      // expects.  Each thread keeps the token ids of its rows in registers
      // (no barrier between the gather warps, so an aborted wait in one
      // cannot strand the others) and ends each stage with an mbarrier
      // arrival that fires when its copies land, so a stage is published as
      // soon as its bytes are in shared memory.  cp.async writes through the
      // generic proxy: the MMA thread fences the proxies after its wait.
      constexpr int kRows = (BT + 11) / 12;     // rows per thread
      const int gw = warp == 0 ? 0 : warp - 1;  // gather warp 0..2
      const int chunk = lane & 7;
      const int r0 = 4 * gw + (lane >> 3);
      for (int64_t t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
        const TileInfo ti = tile_info(t, off_s, ts_s, E, BT, NS);
        int32_t tk[kRows];
#pragma unroll
        for (int i = 0; i < kRows; ++i) {
          const int r = r0 + 12 * i;
          tk[i] = r < ti.nv ? token_of_row(pb.row_to_token, ti.p0 + r, pb.T, pb.err) : -1;
        }
        for (int kb = 0; kb < NK; ++kb, ++g) {
          const uint32_t s = g % XS, ph = (g / XS) & 1u;
          if (!(ok = __all_sync(0xffffffffu, mbar_wait(&x_empty[s], ph ^ 1u, abort, pb.err)))) break;
          const uint32_t dst = smem_u32(smem + Smem::x + s * kXStageBytes);
          const uint16_t* xk = pb.x + kb * BK + chunk * 8;
          if (!kTail || kb * BK + chunk * 8 < K) {
#pragma unroll
            for (int i = 0; i < kRows; ++i) {
              const int r = r0 + 12 * i;
              if (tk[i] >= 0)
                cp_async_16(dst + r * 128 + ((chunk ^ (r & 7)) << 4), xk + (int64_t)tk[i] * K);
            }
          } else {  // past the row's end in a half last stage: zeros
            for (int i = 0; i < kRows; ++i) {
              const int r = r0 + 12 * i;
              if (tk[i] >= 0) cp_async_16_fill(dst + r * 128 + ((chunk ^ (r & 7)) << 4), pb.x, 0u);
            }
          }
          cp_async_arrive_noinc(&x_full[s]);
        }
      }
      cp_async_wait_all();  // nothing may still be landing when the CTA exits
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    // One thread keeps the tensor core fed: the loop holds no descriptor
    // arithmetic beyond 64-bit adds (the start-address field counts 16-byte
    // units), because everything this thread executes between MMAs adds to
    // their issue time (measured: a 128 x 256 x 16 MMA takes 128 cycles when
    // issued back to back, ~240 with descriptors rebuilt around it).
    if (lane == 0) {
      uint32_t g = 0;
      bool ok = true;
      const uint64_t xdesc0 = make_sdesc_sw128(smem_u32(smem + Smem::x), 16, 1024);
      const uint64_t adesc0 = make_sdesc_sw128(smem_u32(smem + Smem::a), 16, 1024);
      AccSched acc;
      for (int64_t t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
        const TileInfo ti = tile_info(t, off_s, ts_s, E, BT, NS);
        const bool wide = ti.nv > BH;
        const uint32_t h0 = acc.h, h1 = acc.h ^ 1u;
        const uint32_t idesc0 = make_idesc_bf16(BM, wide ? (uint32_t)BH : (uint32_t)((ti.nv + 15) & ~15), 0, 0);
        const uint32_t idesc1 = make_idesc_bf16(BM, (uint32_t)((ti.nv - BH + 15) & ~15), 0, 0);
        if (!(ok = mbar_wait(&acc_empty[h0], acc.phase(h0) ^ 1u, abort, pb.err))) break;
        tc_fence_after();
        // a wide tile's second half is waited for just before its first MMA,
        // so the first stage's MMAs into h0 run while the epilogue still
        // drains h1
        bool h1_free = !wide;
        const uint32_t d0 = tmem + h0 * 256u, d1 = tmem + h1 * 256u;
        for (int kb = 0; kb < NK; ++kb, ++g) {
          const uint32_t xs = g % XS, as = g % AS;
          if (!(ok = mbar_wait(&a_full[as], (g / AS) & 1u, abort, pb.err))) break;
          if (!(ok = mbar_wait(&x_full[xs], (g / XS) & 1u, abort, pb.err))) break;
          if (gathered) fence_proxy_async();  // cp.async landed via the generic proxy
          tc_fence_after();
          const uint64_t ad = adesc0 + (uint64_t)((as * kAStageBytes) >> 4);
          const uint64_t bd = xdesc0 + (uint64_t)((xs * kXStageBytes) >> 4);
          // one decoded A stage feeds both halves of a wide tile
          tc_mma_ss(d0, ad, bd, idesc0, kb != 0);
          tc_mma_ss(d0, ad + 2, bd + 2, idesc0, 1u);  // +32 bytes: next 16 K
          tc_mma_ss(d0, ad + 4, bd + 4, idesc0, 1u);
          tc_mma_ss(d0, ad + 6, bd + 6, idesc0, 1u);
          if (wide) {
            if (!h1_free) {
              if (!(ok = mbar_wait(&acc_empty[h1], acc.phase(h1) ^ 1u, abort, pb.err))) break;
              tc_fence_after();
              h1_free = true;
            }
            const uint64_t bd1 = bd + (uint64_t)(kXHalfBytes >> 4);
            tc_mma_ss(d1, ad, bd1, idesc1, kb != 0);
            tc_mma_ss(d1, ad + 2, bd1 + 2, idesc1, 1u);
            tc_mma_ss(d1, ad + 4, bd1 + 4, idesc1, 1u);
            tc_mma_ss(d1, ad + 6, bd1 + 6, idesc1, 1u);
          }
          tc_commit(&x_empty[xs]);
          tc_commit(&a_empty[as]);
        }
        if (!ok) break;
        tc_commit(&acc_full[h0]);
        if (wide) tc_commit(&acc_full[h1]);
        acc.next(wide);
      }
      // every MMA this thread issued has finished before TMEM is released
      tc_commit(mma_done);
      mbar_drain(mma_done, 0);
    }
  } else if (warp >= 4 && warp < 12) {
    // ---------------- decode ----------------
    // Group grp (warps 4-7 or 8-11) takes the stages g = grp + 2h.  The
    // packed bytes of a stage (128 rows x 32 bytes) arrive by TMA into the
    // group's own ring: the first lane of the group issues stage h + WG once
    // all four warps have read slot h.  A tile's scales (128 consecutive
    // rows of one expert: one contiguous range) arrive by one bulk copy
    // into a double buffer, issued a tile ahead by the first lane of group
    // 0; shapes whose tile scales do not fit load each stage's scale per
    // thread instead, two stages ahead.
    // These warps bound the kernel by the instructions they issue, so the
    // loop keeps its bookkeeping incremental: a cursor per look-ahead
    // distance (the stage being decoded, the scale load, the weight TMA)
    // steps two stages at a time and looks a tile up only when it enters a
    // new one -- no divisions per stage.
    const uint32_t grp = (uint32_t)(warp - 4) >> 2;
    const uint32_t q = (uint32_t)warp & 3u;
    const int m = (int)(q * 32 + lane);              // weight row in tile
    // A-tile row of weight row m: SwiGLU puts gate j at 32*(j/16) + j%16 and
    // up j sixteen rows further (lanes l and l + 16 of one epilogue warp)
    const int ar = kGLU ? ((m & 63) >> 4) * 32 + ((m >> 6) << 4) + (m & 15) : m;
    const int mr = ar & 7;                           // row inside its 8-row atom
    const bool issuer = q == 0 && lane == 0;         // packed-weight TMA
    const bool sc_issuer = issuer && grp == 0;       // tile-scale copies
    uint64_t* wf = w_full + grp * WG;
    uint64_t* we = w_empty + grp * WG;
    uint8_t* wring = smem + Smem::w + grp * WG * kWStageBytes;
    const int64_t my_tiles = blockIdx.x < ntiles ? (ntiles - 1 - blockIdx.x) / gridDim.x + 1 : 0;
    const uint32_t total = (uint32_t)(my_tiles * NK);
    const uint32_t nh = total > grp ? (total - grp + 1) / 2 : 0;  // this group's stages
    // first weight row (e * N + n0) of local tile tl
    auto tile_row = [&](int64_t tl) -> int64_t {
      const TileInfo ti = tile_info(blockIdx.x + tl * gridDim.x, off_s, ts_s, E, BT, NS);
      return (int64_t)ti.e * N + ti.n0;
    };
    auto tile_n0 = [&](int64_t tl) -> int32_t {
      return tile_info(blockIdx.x + tl * gridDim.x, off_s, ts_s, E, BT, NS).n0;
    };
    // cursor: local tile tl and stage kb of group stage h; step() = h + 1
    struct Cursor {
      int64_t tl;
      int kb;
    };
    auto at = [&](uint32_t hh) -> Cursor {  // once per cursor, at the start
      const uint32_t g = grp + 2 * hh;
      return Cursor{(int64_t)(g / NK), (int)(g % NK)};
    };
    auto step = [&](Cursor& c) -> bool {  // true when it enters a new tile
      c.kb += 2;
      if (c.kb < NK) return false;
      do { c.kb -= NK; ++c.tl; } while (c.kb >= NK);
      return true;
    };
    // weight TMA cursor (issuer lane only)
    Cursor wc = at(0);
    int32_t wrow0 = nh ? (int32_t)tile_row(wc.tl) : 0;
    uint32_t issued = 0;  // group stages whose packed bytes were requested
    auto issue_w = [&]() {  // the stage at wc into slot issued % WG
      const uint32_t slot = issued % WG;
      ++issued;
      mbar_arrive_expect_tx(&wf[slot], kWStageBytes);
      if (kGLU) {  // 64 gate rows, then the matching 64 up rows
        tma_load_2d(wring + slot * kWStageBytes, &tmw64, wc.kb * (BK / 2), wrow0, &wf[slot]);
        tma_load_2d(wring + slot * kWStageBytes + kWStageBytes / 2, &tmw64, wc.kb * (BK / 2),
                    wrow0 + glu_i, &wf[slot]);
      } else {
        tma_load_2d(wring + slot * kWStageBytes, &tmw, wc.kb * (BK / 2), wrow0, &wf[slot]);
      }
      if (step(wc) && issued < nh) wrow0 = (int32_t)tile_row(wc.tl);
    };
    // one tile's scales: rows e*N + n0 .. +127 (clipped at the end of the
    // array); rows past the expert are read but never used
    const int64_t total_rows = (int64_t)E * N;
    int64_t sc_issued = 0;
    auto issue_sc = [&](int64_t tl) {
      const int64_t row0 = tile_row(tl);
      sc_issued = tl + 1;
      const uint8_t* sbase = reinterpret_cast<const uint8_t*>(pb.scale);
      uint8_t* sdst = smem + Smem::sc + (tl & 1) * kScaleBuf;
      if (kGLU) {  // the gate rows' scales, then the up rows'
        const uint32_t half = (uint32_t)(64 * srow);
        mbar_arrive_expect_tx(&sc_full[tl & 1], 2 * half);
        bulk_load(sdst, sbase + row0 * srow, half, &sc_full[tl & 1]);
        bulk_load(sdst + half, sbase + (row0 + glu_i) * srow, half, &sc_full[tl & 1]);
      } else {
        const int64_t rows = min((int64_t)BM, total_rows - row0);
        const uint32_t bytes = (uint32_t)(rows * srow);
        mbar_arrive_expect_tx(&sc_full[tl & 1], bytes);
        bulk_load(sdst, sbase + row0 * srow, bytes, &sc_full[tl & 1]);
      }
    };
    // per-thread scale loads (when tile scales do not fit): cursor two
    // stages ahead of the decode and this thread's scale row of its tile
    Cursor lc = at(0);
    const uint8_t* lrow = nullptr;  // scale row of weight row m, or null past N
    const int sbytes = F == Fmt::NF4 ? 4 : 2;  // scale bytes per stage
    auto lrow_of = [&](int64_t tl) -> const uint8_t* {
      if (kGLU)  // gate row n0 + m, or up row glu_i + n0 + m - 64
        return reinterpret_cast<const uint8_t*>(pb.scale) +
               (tile_row(tl) + (m < 64 ? m : glu_i + m - 64)) * (int64_t)srow;
      const int32_t n0 = tile_n0(tl);
      if (n0 + m >= N) return nullptr;
      return reinterpret_cast<const uint8_t*>(pb.scale) + (tile_row(tl) + m) * (int64_t)srow;
    };
    auto scale_next = [&](uint32_t hh) -> uint32_t {  // the scale of stage hh (= lc)
      uint32_t v = 0;
      if (hh < nh) {
        if (lrow) {
          if (F == Fmt::NF4) {
            v = __ldg(reinterpret_cast<const uint32_t*>(lrow + lc.kb * sbytes));
          } else if (!kTail || !(srow & 1)) {
            v = __ldg(reinterpret_cast<const uint16_t*>(lrow + lc.kb * sbytes));
          } else {
            // odd rows of scales (K % 64 == 32): byte loads, and the half
            // stage past the row's end decodes with scale byte 127 (2^0)
            const uint8_t* p = lrow + lc.kb * sbytes;
            v = (uint32_t)__ldg(p) | (lc.kb + 1 < NK ? (uint32_t)__ldg(p + 1) << 8 : 127u << 8);
          }
        }
        if (step(lc) && hh + 1 < nh) lrow = lrow_of(lc.tl);
      }
      return v;
    };
    if (issuer)
      while (issued < WG && issued < nh) issue_w();
    if (sc_issuer && tile_scales)
      for (int64_t t = 0; t < 2 && t < my_tiles; ++t) issue_sc(t);
    uint32_t sA = 0, sB = 0;
    if (!tile_scales) {
      if (nh) lrow = lrow_of(lc.tl);
      sA = scale_next(0);
      sB = scale_next(1);
    }
    bool ok = true;
    uint32_t h = 0;  // next group stage
    Cursor dc = at(0);  // the stage being decoded
    auto publish_slot = [&](uint32_t slot) {
      fence_proxy_async();  // generic-proxy stores -> tensor core reads
      __syncwarp();
      if (lane == 0) mbar_arrive(&a_full[slot]);
    };
    uint32_t ws = 0, wph = 0;              // packed-weight slot and parity of stage h
    uint32_t as = grp, aph = 0;            // A slot and parity of stage h
    auto stage = [&](uint32_t sv) -> bool {
      const int64_t tl = dc.tl;
      const int kb = dc.kb;
      if (tile_scales && kb < 2) {  // the group's first stage of this tile
        if (!__all_sync(0xffffffffu, mbar_wait(&sc_full[tl & 1], (uint32_t)(tl >> 1) & 1u, abort, pb.err)))
          return false;
        // the other buffer: its tile (tl - 1) must be released by both groups
        bool good = true;
        if (sc_issuer && tl >= 1 && tl + 1 < my_tiles) {
          good = mbar_wait(&sc_empty[(tl + 1) & 1], (uint32_t)((tl - 1) >> 1) & 1u, abort, pb.err);
          if (good) issue_sc(tl + 1);
        }
        if (!__all_sync(0xffffffffu, good)) return false;
      }
      if (!__all_sync(0xffffffffu, mbar_wait(&wf[ws], wph, abort, pb.err))) return false;
      const uint8_t* wrow_s = wring + ws * kWStageBytes + m * 32;
      const uint4 q0 = *reinterpret_cast<const uint4*>(wrow_s);
      const uint4 q1 = *reinterpret_cast<const uint4*>(wrow_s + 16);
      if (tile_scales) {
        const uint8_t* sb = smem + Smem::sc + (tl & 1) * kScaleBuf + m * srow + kb * sbytes;
        sv = F == Fmt::NF4 ? *reinterpret_cast<const uint32_t*>(sb)
                           : (uint32_t)*reinterpret_cast<const uint16_t*>(sb);
      }
      const uint32_t P[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
      uint32_t o[32];
      if (F == Fmt::NF4) {
        const Planes tb = nf4_planes(__uint_as_float(sv));
#pragma unroll
        for (int i = 0; i < 8; ++i) decode_word<true>(P[i], tb, &o[4 * i]);
      } else {
        const Planes t0 = mxfp4_planes(sv & 0xFFu);
#pragma unroll
        for (int i = 0; i < 4; ++i) decode_word<false>(P[i], t0, &o[4 * i]);
        const Planes t1 = mxfp4_planes((sv >> 8) & 0xFFu);
#pragma unroll
        for (int i = 4; i < 8; ++i) decode_word<false>(P[i], t1, &o[4 * i]);
      }
      // Release the packed-weight slot (and, after the tile's last stage,
      // the scale buffer) only now that the decode has consumed the values
      // loaded from them: the refill is an async-proxy write, and releasing
      // right after issuing the shared-memory loads let the refill of the
      // issuing warp's own slot overtake loads still in flight.
      __syncwarp();
      if (lane == 0) mbar_arrive(&we[ws]);
      if (tile_scales && kb + 2 >= NK && lane == 0) mbar_arrive(&sc_empty[tl & 1]);
      bool good = true;
      if (issuer && issued < nh) {
        // slot ws is free once all four warps of the group have used it
        good = mbar_wait(&we[ws], wph, abort, pb.err);
        if (good) issue_w();
      }
      if (!__all_sync(0xffffffffu, good)) return false;
      if (!__all_sync(0xffffffffu, mbar_wait(&a_empty[as], aph ^ 1u, abort, pb.err))) return false;
      // row m of the K-major, 128B-swizzled A tile: chunk c at (c ^ (m % 8))
      uint8_t* dst = smem + Smem::a + as * kAStageBytes + ar * 128;
#pragma unroll
      for (int c = 0; c < 8; ++c)
        *reinterpret_cast<uint4*>(dst + ((c ^ mr) << 4)) =
            make_uint4(o[4 * c], o[4 * c + 1], o[4 * c + 2], o[4 * c + 3]);
      publish_slot(as);
      // next group stage: slots advance by one (weights) and two (A)
      if (++ws == WG) { ws = 0; wph ^= 1u; }
      as += 2;
      if (as >= AS) { as -= AS; aph ^= 1u; }
      step(dc);
      return true;
    };
    // unrolled by two with one scale register per half: the scale of stage
    // h + 2 is loaded right after stage h and not read until then (a queue
    // rotated by register copies would wait on each load right away)
    while (h < nh) {
      if (!(ok = stage(sA))) break;
      ++h;
      if (!tile_scales) sA = scale_next(h + 1);
      if (h >= nh) break;
      if (!(ok = stage(sB))) break;
      ++h;
      if (!tile_scales) sB = scale_next(h + 1);
    }
    // After an abort, copies this group requested but did not consume must
    // land before the CTA exits (shared memory is still their target).
    if (issuer && !ok)
      for (uint32_t d = h; d < issued; ++d) mbar_drain(&wf[d % WG], (d / WG) & 1u);
    if (sc_issuer && !ok)
      for (int64_t t = (sc_issued > 2 ? sc_issued - 2 : 0); t < sc_issued; ++t)
        mbar_drain(&sc_full[t & 1], (uint32_t)(t >> 1) & 1u);
  } else if (warp >= 12) {
    // ---------------- epilogue ----------------
    // Thread t of warp q holds output column n0 + 32q + t for 32 routed rows
    // per TMEM chunk; a 32 x 32 bf16 transpose through shared memory turns
    // that into 64 contiguous bytes of one output row per thread, written
    // with four 16-byte stores.  A wide tile's halves are drained in order,
    // each released as soon as it has been read.
    const uint32_t q = (uint32_t)warp & 3u;
    uint8_t* stage = smem + Smem::epi + q * kEpiWarpBytes;
    AccSched acc;
    bool ok = true;
    for (int64_t t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
      const TileInfo ti = tile_info(t, off_s, ts_s, E, BT, NS);
      const bool wide = ti.nv > BH;
      const int ncol0 = ti.n0 + (int)q * 32;  // first output column of this warp
      const int sub = lane & 3;               // 16-byte piece of a row
      const bool subok = ncol0 + sub * 8 < N;
      for (int part = 0; part < (wide ? 2 : 1) && ok; ++part) {
        const uint32_t hf = part ? acc.h ^ 1u : acc.h;
        const int row0 = part * BH;
        const int rows = part ? ti.nv - BH : min(ti.nv, BH);
        ok = __all_sync(0xffffffffu, mbar_wait(&acc_full[hf], acc.phase(hf), abort, pb.err));
        if (!ok) break;
        tc_fence_after();
        const uint32_t tlane = tmem + ((q * 32u) << 16) + hf * 256u;
        const int nchunks = (rows + 31) >> 5;
        for (int c = 0; c < nchunks; ++c) {
          uint32_t r[32];
          tmem_load_32x32b_x32(tlane + c * 32, r);
          if (c == nchunks - 1) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[hf]);
          }
          if (kGLU) {
            // lane l holds A-tile row 32q + l: gate (l < 16) or up (l >= 16)
            // of h column n0 + 16q + l % 16, for the chunk's 32 routed rows.
            // The two lanes of a column split the rows: the gate lane takes
            // rows 0-15, the up lane rows 16-31, each receiving the other
            // operand by one shuffle.  Both operands are rounded to bf16
            // (the gate_up output); h = bf16(silu(gate) * up) goes into a
            // 32-row x 16-column transpose.
            const bool glane = lane < 16;
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const float mine = __bfloat162float(
                  __float2bfloat16_rn(__uint_as_float(glane ? r[j] : r[j + 16])));
              const float send = __bfloat162float(
                  __float2bfloat16_rn(__uint_as_float(glane ? r[j + 16] : r[j])));
              const float other = __shfl_xor_sync(0xffffffffu, send, 16);
              const float g = glane ? mine : other, u = glane ? other : mine;
              *reinterpret_cast<uint16_t*>(stage + (glane ? j : j + 16) * 32 + (lane & 15) * 2) =
                  __bfloat16_as_ushort(__float2bfloat16_rn(__fdividef(g, 1.0f + __expf(-g)) * u));
            }
            __syncwarp();
            // two lanes write one routed row's 32 bytes of h
#pragma unroll
            for (int v = 0; v < 2; ++v) {
              const int rr = (lane >> 1) + 16 * v;  // row within the chunk
              const int row = c * 32 + rr;
              if (row < rows)
                *reinterpret_cast<uint4*>(pb.out + (int64_t)(ti.p0 + row0 + row) * ON + ti.n0 +
                                          (int)q * 16 + (lane & 1) * 8) =
                    *reinterpret_cast<const uint4*>(stage + rr * 32 + (lane & 1) * 16);
            }
            __syncwarp();
          } else {
          // thread = output column ncol0 + lane, r[j] = routed row c*32 + j
#pragma unroll
          for (int j = 0; j < 32; ++j)
            *reinterpret_cast<uint16_t*>(stage + j * kEpiRowBytes + lane * 2) =
                __bfloat16_as_ushort(__float2bfloat16_rn(__uint_as_float(r[j])));
          __syncwarp();
          // four lanes write one routed row's 64 bytes, so each store
          // instruction covers eight whole row segments (full 32-byte sectors)
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            const int rr = (lane >> 2) + 8 * v;  // row within the chunk
            const int row = c * 32 + rr;         // routed row within the half
            if (row < rows && subok)
              *reinterpret_cast<uint4*>(pb.out + (int64_t)(ti.p0 + row0 + row) * ON + ncol0 + sub * 8) =
                  *reinterpret_cast<const uint4*>(stage + rr * kEpiRowBytes + sub * 16);
          }
          __syncwarp();
          }
        }
      }
      acc.next(wide);
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

static_assert(1024 + Smem::tables + 8 * (1024 + 1) <= 232448,
              "shared memory for 1024 experts exceeds the 227 KB a CTA can have");

size_t gemm_smem_bytes(int32_t E) {
  return 1024 + Smem::tables + sizeof(int32_t) * 2 * (size_t)(E + 1);
}

cudaError_t launch_gemm(Fmt f, const GroupedProblem& pb, int num_sms,
                        cudaStream_t s, int64_t glu_i) {
  if (pb.P == 0 || pb.N == 0) return cudaSuccess;
  CUtensorMap tmx;
  // identity rows: boxes of 64 K x 256 rows (one per tile half); gathered rows use cp.async and
  // never read this map
  cudaError_t e = make_map_2d(&tmx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, pb.x,
                              (uint64_t)pb.K, (uint64_t)(pb.T > 0 ? pb.T : 1),
                              (uint64_t)pb.K * 2, BK, BH, CU_TENSOR_MAP_SWIZZLE_128B);
  if (e != cudaSuccess) return e;
  CUtensorMap tmx32;  // the same rows in boxes of 32, for partial tiles
  e = make_map_2d(&tmx32, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, pb.x,
                  (uint64_t)pb.K, (uint64_t)(pb.T > 0 ? pb.T : 1),
                  (uint64_t)pb.K * 2, BK, 32, CU_TENSOR_MAP_SWIZZLE_128B);
  if (e != cudaSuccess) return e;
  // packed weights [E*N rows, K/2 bytes]: boxes of 32 bytes (one 64-K stage)
  // x 128 rows (x 64 rows for the SwiGLU tiles' gate and up halves); rows
  // past E*N read as zeros
  CUtensorMap tmw, tmw64;
  e = make_map_2d(&tmw, CU_TENSOR_MAP_DATA_TYPE_UINT8, pb.w, (uint64_t)pb.K / 2,
                  (uint64_t)pb.E * (uint64_t)pb.N, (uint64_t)pb.K / 2, BK / 2, BM,
                  CU_TENSOR_MAP_SWIZZLE_NONE);
  if (e != cudaSuccess) return e;
  e = make_map_2d(&tmw64, CU_TENSOR_MAP_DATA_TYPE_UINT8, pb.w, (uint64_t)pb.K / 2,
                  (uint64_t)pb.E * (uint64_t)pb.N, (uint64_t)pb.K / 2, BK / 2, 64,
                  CU_TENSOR_MAP_SWIZZLE_NONE);
  if (e != cudaSuccess) return e;
  // A tile's scales (128 rows x srow bytes, contiguous; for SwiGLU tiles two
  // ranges of 64 rows) come by bulk copy when they fit the buffer, there are
  // at least two stages per tile (so both decode groups take part in every
  // tile) and every copy stays 16-byte aligned: rows start at multiples of
  // 64, so N * srow, glu_i * srow and the array's address must be multiples
  // of 16; srow must be even, since the decode reads two MXFP4 scale bytes as
  // one 16-bit word (K % 64 == 32 leaves it odd: per-thread byte loads).
  const int srow = (f == Fmt::NF4) ? (int)(pb.K / 64) * 4 : (int)(pb.K / 32);
  const int tile_scales = (pb.K / BK >= 2) && (BM * srow <= kScaleBuf) && (srow % 2 == 0) &&
                          ((pb.N * srow) % 16 == 0) && ((64 * (int64_t)srow) % 16 == 0) &&
                          ((glu_i * srow) % 16 == 0) &&
                          (reinterpret_cast<uintptr_t>(pb.scale) % 16 == 0);
  const size_t smem = gemm_smem_bytes(pb.E);
  // wide tiles when activations come by TMA (identity rows), narrow when
  // they are gathered through row_to_token
  const bool wide = pb.row_to_token == nullptr;
  const bool glu = glu_i > 0;
  using KFn = void (*)(const GroupedProblem, const CUtensorMap, const CUtensorMap,
                       const CUtensorMap, const CUtensorMap, const int, const int, const int32_t);
  KFn k;
#define GBW_GEMM_PICK(FF)                                                              \
  k = glu ? (wide ? gemm_kernel<FF, true, true> : gemm_kernel<FF, false, true>)        \
          : (wide ? gemm_kernel<FF, true, false> : gemm_kernel<FF, false, false>);
  if (f == Fmt::NF4) { GBW_GEMM_PICK(Fmt::NF4) } else { GBW_GEMM_PICK(Fmt::MXFP4) }
#undef GBW_GEMM_PICK
  e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem);
  if (e != cudaSuccess) return e;
  k<<<num_sms, kThreads, smem, s>>>(pb, tmx, tmx32, tmw, tmw64, srow, tile_scales,
                                     (int32_t)glu_i);
  return cudaGetLastError();
}

}  // namespace gbw
