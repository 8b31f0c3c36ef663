/*
 * gbw.h -- C ABI of the B200 grouped 4-bit MoE matmul library (libgbw.so).
 *
 * One call multiplies bf16 activations by the 4-bit packed weights of every
 * active expert ("grouped-nf4-gemm 0.43.0" project page, opening lines: one
 * GPU launch for the active experts, no full-size bf16 weight copies;
 * "Receipts-driven engineering", opening paragraph: the codebook is decoded
 * in registers inside the GEMM mainloop, NF4 in the bitsandbytes packed
 * format unchanged, MXFP4 as OCP e2m1 on released checkpoint bytes, the NF4
 * path differentiable).
 *
 * Conventions for every entry point
 *  - All array arguments are DEVICE pointers owned by the caller; the library
 *    never allocates, frees or keeps them.  Inputs are only read.
 *  - bf16 arrays are passed as uint16_t bit patterns.
 *  - `stream` is a cudaStream_t (NULL = the legacy default stream).  Every
 *    call is asynchronous on that stream and does no host synchronisation.
 *  - Host-side checks (NULL pointers, sizes, alignment, device architecture)
 *    return an error code before anything is launched.
 *  - Checks that need device data (expert_offsets, row_to_token) run inside
 *    the kernels: offsets are clamped to a running maximum in [0, P] and
 *    token indices to [0, T), so no access leaves the caller's buffers; the
 *    violation is recorded in a per-device error word that
 *    gbw_device_status() reads.  The same word records a bounded wait that
 *    gave up (the kernel then returns instead of hanging).
 *  - The library runs only on sm_100 devices (B200); anything else returns
 *    GBW_ERR_ARCH.  There is no fallback path.
 */
#ifndef GBW_H_
#define GBW_H_

#include <stdint.h>

#if defined(__GNUC__)
#define GBW_API __attribute__((visibility("default")))
#else
#define GBW_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  GBW_OK = 0,
  GBW_ERR_NULL = 1,   /* a required pointer is NULL */
  GBW_ERR_SHAPE = 2,  /* a size is negative or breaks a divisibility rule */
  GBW_ERR_ALIGN = 3,  /* a pointer or row stride is not 16-byte aligned */
  GBW_ERR_ARCH = 4,   /* the current device is not sm_100 */
  GBW_ERR_LAUNCH = 5, /* a CUDA call failed (cudaGetLastError text kept) */
  GBW_ERR_DEVICE = 6  /* gbw_device_status found a device-side error */
} gbw_status;

typedef enum {
  GBW_MODE_AUTO = 0, /* GEMV when P <= 4 * E (at most ~4 routed rows per
                        expert on average), else the tensor-core GEMM */
  GBW_MODE_GEMM = 1, /* force the tcgen05 grouped GEMM */
  GBW_MODE_GEMV = 2  /* force the bandwidth GEMV (no tensor cores) */
} gbw_mode;

/* Flag OR-ed into the mode argument of the grouped forward calls.
 * GBW_FLAG_OVERLAP_PREV: the caller guarantees that the packed weights, the
 * scales, expert_offsets and row_to_token of this call are not written by
 * the kernel launched immediately before it on the same stream (in a MoE
 * layer they come from the checkpoint and the router, launched earlier).
 * The bandwidth GEMV then reads them while that kernel is still finishing
 * (programmatic dependent launch); it reads x and writes out only after the
 * preceding kernel has completed, with or without the flag.  Passing the
 * flag when the guarantee does not hold gives undefined results. */
#define GBW_FLAG_OVERLAP_PREV 0x100

/* Bits of the device error word. */
#define GBW_DEVERR_OFFSETS 1 /* expert_offsets not 0 <= ... <= P (clamped) */
#define GBW_DEVERR_TOKEN 2   /* row_to_token[p] outside [0, T) (clamped) */
#define GBW_DEVERR_TIMEOUT 4 /* a pipeline wait gave up; output incomplete */

/* Grouped NF4 forward ("grouped-nf4-gemm 0.43.0", "Which entry point?":
 * nf4_grouped.gemm_4bit_grouped; the bandwidth route of the 0.43.0 notes is
 * GBW_MODE_GEMV).
 *   out[p, n] = bf16( sum_k x[tok(p), k] * W_e(p)[n, k] ),  fp32 accumulation
 *   W_e[n, k] = NF4[q] * absmax[e, n, k/64]  (q = code of element k)
 *   x              [T, K]   bf16, row-major
 *   packed         [E, N, K/2] uint8: byte j of a row holds elements 2j (high
 *                  nibble) and 2j+1 (low nibble) -- the bitsandbytes layout
 *   absmax         [E, N, K/64] fp32, one per 64 consecutive K elements
 *   expert_offsets [E+1] int32 (device): routed rows are sorted by expert;
 *                  rows expert_offsets[e] .. expert_offsets[e+1]-1 use expert
 *                  e; expert_offsets[0] = 0, expert_offsets[E] = P
 *   row_to_token   [P] int32 (device) or NULL: routed row p reads x row
 *                  row_to_token[p]; NULL means row p reads x row p (T >= P)
 *   out            [P, N] bf16, row-major, expert-sorted row order
 * mode           a gbw_mode, optionally OR-ed with GBW_FLAG_OVERLAP_PREV
 * Requires K % 64 == 0, N % 8 == 0, 1 <= E <= 1024, and 16-byte aligned x,
 * packed and out.  P == 0 is a no-op.  Experts with no rows cost nothing. */
GBW_API gbw_status gnf4_grouped_gemm(const uint16_t* x, int64_t T, int64_t K,
                             const uint8_t* packed, const float* absmax,
                             int32_t E, int64_t N,
                             const int32_t* expert_offsets,
                             const int32_t* row_to_token, int64_t P,
                             uint16_t* out, int32_t mode, void* stream);

/* Grouped MXFP4 forward ("grouped-nf4-gemm 0.43.0", "Which entry point?":
 * mxfp4_grouped.gemm_mxfp4_grouped; "native MXFP4 MoE inference": e2m1
 * blocks with e8m0 scales, no requantisation, no bf16 materialisation).
 *   W_e[n, k] = e2m1(code) * 2^(scales[e, n, k/32] - 127)
 *   blocks [E, N, K/32, 16] uint8 (= [E, N, K/2]): byte j holds elements 2j
 *          (LOW nibble) and 2j+1 (high nibble); bit 3 of a code is its sign
 *   scales [E, N, K/32] uint8, e8m0 (0xFF is NaN), 2-byte aligned
 * Everything else as gnf4_grouped_gemm; requires K % 32 == 0, N % 8 == 0.
 * K % 64 == 32 is taken by both paths: the tensor-core GEMM runs its last
 * 64-wide K stage half full, zeros in the upper half on both operands. */
GBW_API gbw_status gmxfp4_grouped_gemm(const uint16_t* x, int64_t T, int64_t K,
                               const uint8_t* blocks, const uint8_t* scales,
                               int32_t E, int64_t N,
                               const int32_t* expert_offsets,
                               const int32_t* row_to_token, int64_t P,
                               uint16_t* out, int32_t mode, void* stream);

/* Grouped NF4 activation gradient ("grouped-nf4-gemm 0.43.0", "Which entry
 * point?": dgrad_4bit_grouped; "Receipts-driven engineering": fine-tuning
 * never leaves the packed format).
 *   dx[p, k] = bf16( sum_n dy[p, n] * W_e(p)[n, k] ),  fp32 accumulation
 *   dy [P, N] bf16 row-major (expert-sorted rows), dx [P, K] bf16 row-major;
 *   packed / absmax / expert_offsets exactly as in gnf4_grouped_gemm (the
 *   weights are read packed, in the transposed orientation).
 * Requires K % 64 == 0, N % 64 == 0, 16-byte aligned dy, packed and dx. */
GBW_API gbw_status gnf4_grouped_dgrad(const uint16_t* dy, int64_t P, int64_t N,
                              const uint8_t* packed, const float* absmax,
                              int32_t E, int64_t K,
                              const int32_t* expert_offsets, uint16_t* dx,
                              void* stream);

/* Grouped MXFP4 activation gradient ("grouped-nf4-gemm 0.43.0", "Which
 * entry point?": the MXFP4 entry point; "Receipts-driven engineering":
 * training on the released MXFP4 bytes without requantisation).
 *   dx[p, k] = bf16( sum_n dy[p, n] * W_e(p)[n, k] ),  fp32 accumulation
 *   dy, dx, expert_offsets as in gnf4_grouped_dgrad; blocks / scales as in
 *   gmxfp4_grouped_gemm (read packed, in the transposed orientation).
 * Requires K % 64 == 0, N % 64 == 0, 16-byte aligned dy, blocks and dx,
 * 2-byte aligned scales. */
GBW_API gbw_status gmxfp4_grouped_dgrad(const uint16_t* dy, int64_t P, int64_t N,
                                const uint8_t* blocks, const uint8_t* scales,
                                int32_t E, int64_t K,
                                const int32_t* expert_offsets, uint16_t* dx,
                                void* stream);

/* Fused expert pass, NF4 ("Receipts-driven engineering", "The numbers":
 * the fused training row over all 48 Qwen3-30B-A3B layers -- the expert
 * MLP runs gate_up, the SwiGLU combine and down in one pass per routed row).
 *   gate_up[p, :] = x[tok(p)] @ Wgu_e(p)^T          (2I columns, bf16)
 *   h[p, j]       = bf16( silu(gate_up[p, j]) * gate_up[p, I + j] ),
 *                   silu(v) = v / (1 + e^-v), evaluated in fp32
 *   out[p, :]     = h[p] @ Wdn_e(p)^T                (H columns, bf16)
 * The page names the pass but prints neither the activation nor the
 * gate/up layout; the reading taken is the standard SwiGLU with the gate
 * rows [0, I) stacked above the up rows [I, 2I) of each expert's gate_up
 * weight.
 *   x          [T, H] bf16 row-major; row_to_token / expert_offsets / P as
 *              in gnf4_grouped_gemm
 *   gu_packed  [E, 2I, H/2] uint8, gu_absmax [E, 2I, H/64] fp32
 *   dn_packed  [E, H, I/2] uint8, dn_absmax [E, H, I/64] fp32
 *   h          [P, I] bf16 WORKSPACE supplied by the caller: written by the
 *              gate_up kernel, read by the down kernel (it keeps h)
 *   out        [P, H] bf16, expert-sorted row order
 *   mode       AUTO: both projections on the bandwidth GEMV when P <= 4 * E,
 *              else both on the tensor cores; GEMM / GEMV force a path.  No
 *              flags.  SwiGLU is computed where the gate and up sums meet
 *              (the GEMM epilogue pairs them in one tile, the GEMV in one
 *              warp), so gate_up is never written out.
 * Requires H % 64 == 0, I % 64 == 0, 16-byte aligned x, weights, h and out.
 * Two kernels are launched on `stream`, in order. */
GBW_API gbw_status gnf4_grouped_expert_mlp(const uint16_t* x, int64_t T, int64_t H,
                                   const uint8_t* gu_packed, const float* gu_absmax,
                                   const uint8_t* dn_packed, const float* dn_absmax,
                                   int32_t E, int64_t I, const int32_t* expert_offsets,
                                   const int32_t* row_to_token, int64_t P, uint16_t* h,
                                   uint16_t* out, int32_t mode, void* stream);

/* Fused expert pass, MXFP4 (gate_up blocks [E, 2I, H/32, 16] + scales
 * [E, 2I, H/32]; down blocks [E, H, I/32, 16] + scales [E, H, I/32], e8m0,
 * 2-byte aligned).  Everything else as gnf4_grouped_expert_mlp. */
GBW_API gbw_status gmxfp4_grouped_expert_mlp(const uint16_t* x, int64_t T, int64_t H,
                                     const uint8_t* gu_blocks, const uint8_t* gu_scales,
                                     const uint8_t* dn_blocks, const uint8_t* dn_scales,
                                     int32_t E, int64_t I, const int32_t* expert_offsets,
                                     const int32_t* row_to_token, int64_t P, uint16_t* h,
                                     uint16_t* out, int32_t mode, void* stream);

/* Fused NF4 expert pass that allocates nothing and takes no workspace.
 * This entry point has no counterpart on the source pages; it exists for
 * callers that cannot hand the library device memory at call time -- for
 * example a plugin running inside an inference engine that has already
 * reserved all device memory for itself, or a serving loop that forbids
 * allocation after warm-up (cudaMalloc may synchronise the device and
 * fragment memory held by a caching allocator).
 *   Same arguments and results as gnf4_grouped_expert_mlp, without h: the h
 *   rows go to a fixed scratch array inside the library's device image
 *   (4 MiB, which every device that loads the library keeps until the
 *   process exits).
 *   Limit: P * I <= 2,097,152; larger problems return GBW_ERR_SHAPE.
 *   The first call on a device looks up the scratch address for that device
 *   (cudaGetSymbolAddress); make that first call before any stream capture.
 *   All calls share the one array: calls whose kernels may overlap on the
 *   GPU (different streams, or several host threads) race on it and must be
 *   ordered by the caller.  No call depends on what an earlier call left
 *   there.  No device memory is allocated or freed. */
GBW_API gbw_status gnf4_grouped_expert_mlp_noalloc(const uint16_t* x, int64_t T, int64_t H,
                                           const uint8_t* gu_packed, const float* gu_absmax,
                                           const uint8_t* dn_packed, const float* dn_absmax,
                                           int32_t E, int64_t I, const int32_t* expert_offsets,
                                           const int32_t* row_to_token, int64_t P,
                                           uint16_t* out, int32_t mode, void* stream);

/* Decode packed weights to bf16 ("grouped-nf4-gemm 0.43.0", "Try the
 * packers and byte checks on CPU", example 1: dequant_ref).  Bit-exact:
 * w[r, k] = bf16_rn(fp32(NF4[q] * absmax[r, k/64])).  rows counts all
 * expert rows (E*N).  Requires K % 64 == 0 and a 16-byte aligned w_out. */
GBW_API gbw_status gnf4_dequant(const uint8_t* packed, const float* absmax,
                        int64_t rows, int64_t K, uint16_t* w_out,
                        void* stream);

/* MXFP4 decode (same page, example 2: dequant_mxfp4):
 * w[r, k] = bf16_rn(e2m1(code) * 2^(s - 127)).  Requires K % 32 == 0. */
GBW_API gbw_status gmxfp4_dequant(const uint8_t* blocks, const uint8_t* scales,
                          int64_t rows, int64_t K, uint16_t* w_out,
                          void* stream);

/* NF4 packer on the GPU (same page, example 1: quantize_pack_nf4).
 * Per row and 64-block: a = max|w|, q = argmin_i |w/a - NF4[i]| (fp32,
 * lowest index on ties), all-zero block -> a = 0 and code 7.  Byte-identical
 * to the CPU packer.  w [rows, K] fp32; non-finite input is not checked
 * (its codes are unspecified).  Requires K % 64 == 0. */
GBW_API gbw_status gnf4_quantize(const float* w, int64_t rows, int64_t K,
                         uint8_t* packed, float* absmax, void* stream);

/* MXFP4 packer on the GPU (same page, example 2: quantize_pack_mxfp4).
 * Per 32-block: X = floor(log2 max|w|) - 2 clamped to [-127, 127], scale
 * byte X + 127, codes = nearest e2m1 to w / 2^X (ties to even, saturating,
 * sign kept); all-zero block -> scale 0, codes 0.  Requires K % 32 == 0. */
GBW_API gbw_status gmxfp4_quantize(const float* w, int64_t rows, int64_t K,
                           uint8_t* blocks, uint8_t* scales, void* stream);

/* Reads the current device's error word (GBW_DEVERR_* bits) on `stream`,
 * stores it in *host_err, and clears it when `clear` is non-zero.  The word
 * is taken in one atomic step on the device, so a bit that a kernel on
 * another stream raises meanwhile is either returned or kept, never lost.
 * Synchronises `stream`.  Returns GBW_ERR_DEVICE when a bit is set.  Calls
 * for the same device from several host threads at once share one copy
 * slot: serialise them. */
GBW_API gbw_status gbw_device_status(void* stream, int32_t* host_err, int32_t clear);

/* Static text for a status code; the last CUDA error text for
 * GBW_ERR_LAUNCH. */
GBW_API const char* gbw_status_string(gbw_status s);

/* Library version, major * 10000 + minor * 100 + patch. */
GBW_API int32_t gbw_version(void);

#ifdef __cplusplus
}
#endif

#endif /* GBW_H_ */
