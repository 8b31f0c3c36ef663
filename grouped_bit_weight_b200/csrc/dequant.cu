// dequant.cu -- packed 4-bit weights <-> fp32 / bf16 on the GPU.
//
// Decode ("grouped-nf4-gemm 0.43.0", "Try the packers and byte checks on
// CPU": dequant_ref and dequant_mxfp4) writes the bf16 weight that the
// grouped GEMM multiplies: bf16_rn(fp32(code_value * scale)).
// Quantize (same section: quantize_pack_nf4 / quantize_pack_mxfp4) packs
// fp32 weights byte-identically to the CPU packer.
// Both are HBM-streaming kernels: 16-byte loads/stores, grid sized to a
// multiple of the SM count.
#include "common.cuh"

namespace gbw {
namespace {

// The 16-entry NF4 codebook of QLoRA (normal-quantile levels, -1 .. +1).
__constant__ float kNF4[16] = {
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

// OCP e2m1 magnitudes of codes 0..7.
__constant__ float kE2M1[8] = {0.0f, 0.5f, 1.0f, 1.5f, 2.0f, 3.0f, 4.0f, 6.0f};

// 2^(s-127) for an e8m0 byte; 0xFF is NaN.
__device__ __forceinline__ float e8m0_to_f32(uint32_t s) {
  if (s == 0xFFu) return __int_as_float(0x7FC00000);
  if (s == 0u) return __int_as_float(0x00400000);  // 2^-127 (subnormal)
  return __int_as_float((int)(s << 23));
}

__device__ __forceinline__ uint16_t bf16_bits(float v) {
  return __bfloat16_as_ushort(__float2bfloat16_rn(v));
}

// One thread = 16 packed bytes = 32 weights of one row.
__global__ void __launch_bounds__(256) nf4_dequant_kernel(
    const uint8_t* __restrict__ packed, const float* __restrict__ absmax,
    int64_t rows, int64_t K, uint16_t* __restrict__ out) {
  __shared__ float lut[16];
  if (threadIdx.x < 16) lut[threadIdx.x] = kNF4[threadIdx.x];
  __syncthreads();
  const int64_t chunks_per_row = K / 32;
  const int64_t total = rows * chunks_per_row;
  for (int64_t c = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; c < total;
       c += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = c / chunks_per_row, j = c % chunks_per_row;
    const uint4 q = __ldg(reinterpret_cast<const uint4*>(packed + r * (K / 2)) + j);
    const float a = __ldg(absmax + r * (K / 64) + (j >> 1));
    const uint32_t w[4] = {q.x, q.y, q.z, q.w};
    uint32_t o[16];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        const uint32_t byte = (w[i] >> (8 * b)) & 0xFFu;
        const float ev = __fmul_rn(lut[byte >> 4], a);   // even k: high nibble
        const float od = __fmul_rn(lut[byte & 15u], a);  // odd k: low nibble
        o[i * 4 + b] = (uint32_t)bf16_bits(ev) | ((uint32_t)bf16_bits(od) << 16);
      }
    }
    uint4* dst = reinterpret_cast<uint4*>(out + r * K + j * 32);
#pragma unroll
    for (int i = 0; i < 4; ++i)
      dst[i] = make_uint4(o[4 * i], o[4 * i + 1], o[4 * i + 2], o[4 * i + 3]);
  }
}

__global__ void __launch_bounds__(256) mxfp4_dequant_kernel(
    const uint8_t* __restrict__ blocks, const uint8_t* __restrict__ scales,
    int64_t rows, int64_t K, uint16_t* __restrict__ out) {
  __shared__ float lut[16];
  if (threadIdx.x < 16)
    lut[threadIdx.x] = (threadIdx.x & 8) ? -kE2M1[threadIdx.x & 7]
                                         : kE2M1[threadIdx.x & 7];
  __syncthreads();
  const int64_t chunks_per_row = K / 32;
  const int64_t total = rows * chunks_per_row;
  for (int64_t c = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; c < total;
       c += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = c / chunks_per_row, j = c % chunks_per_row;
    const uint4 q = __ldg(reinterpret_cast<const uint4*>(blocks + r * (K / 2)) + j);
    const float sc = e8m0_to_f32(__ldg(scales + r * (K / 32) + j));
    const uint32_t w[4] = {q.x, q.y, q.z, q.w};
    uint32_t o[16];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        const uint32_t byte = (w[i] >> (8 * b)) & 0xFFu;
        const float ev = __fmul_rn(lut[byte & 15u], sc);  // even k: low nibble
        const float od = __fmul_rn(lut[byte >> 4], sc);
        o[i * 4 + b] = (uint32_t)bf16_bits(ev) | ((uint32_t)bf16_bits(od) << 16);
      }
    }
    uint4* dst = reinterpret_cast<uint4*>(out + r * K + j * 32);
#pragma unroll
    for (int i = 0; i < 4; ++i)
      dst[i] = make_uint4(o[4 * i], o[4 * i + 1], o[4 * i + 2], o[4 * i + 3]);
  }
}

// Nearest NF4 code: argmin_i |y - C[i]| in fp32, lowest index on ties.
__device__ __forceinline__ uint32_t nf4_nearest(float y, const float* lut) {
  uint32_t best = 0;
  float bd = fabsf(__fsub_rn(y, lut[0]));
#pragma unroll
  for (uint32_t i = 1; i < 16; ++i) {
    const float d = fabsf(__fsub_rn(y, lut[i]));
    if (d < bd) { bd = d; best = i; }
  }
  return best;
}

// One warp per 64-element block: lane l owns elements 2l and 2l+1.
__global__ void __launch_bounds__(256) nf4_quantize_kernel(
    const float* __restrict__ w, int64_t rows, int64_t K,
    uint8_t* __restrict__ packed, float* __restrict__ absmax) {
  __shared__ float lut[16];
  if (threadIdx.x < 16) lut[threadIdx.x] = kNF4[threadIdx.x];
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int64_t nblocks = rows * (K / 64);
  const int64_t warps = (int64_t)gridDim.x * (blockDim.x / 32);
  for (int64_t b = blockIdx.x * (int64_t)(blockDim.x / 32) + threadIdx.x / 32;
       b < nblocks; b += warps) {
    const float2 v = __ldg(reinterpret_cast<const float2*>(w + b * 64) + lane);
    float m = fmaxf(fabsf(v.x), fabsf(v.y));
#pragma unroll
    for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    uint32_t q0 = 7, q1 = 7;
    if (m > 0.0f) {
      q0 = nf4_nearest(__fdiv_rn(v.x, m), lut);
      q1 = nf4_nearest(__fdiv_rn(v.y, m), lut);
    }
    packed[b * 32 + lane] = (uint8_t)((q0 << 4) | q1);
    if (lane == 0) absmax[b] = m;
  }
}

// Nearest e2m1 magnitude code to v >= 0, ties to the even code.
__device__ __forceinline__ uint32_t e2m1_nearest(float v) {
  uint32_t best = 0;
  float bd = fabsf(__fsub_rn(v, kE2M1[0]));
#pragma unroll
  for (uint32_t c = 1; c < 8; ++c) {
    const float d = fabsf(__fsub_rn(v, kE2M1[c]));
    if (d < bd || (d == bd && (c & 1u) == 0u && (best & 1u) == 1u)) {
      bd = d;
      best = c;
    }
  }
  return best;
}

// Half a warp per 32-element block: lane l of the half owns 2l, 2l+1.
__global__ void __launch_bounds__(256) mxfp4_quantize_kernel(
    const float* __restrict__ w, int64_t rows, int64_t K,
    uint8_t* __restrict__ blocks, uint8_t* __restrict__ scales) {
  const int lane = threadIdx.x & 15;
  const int64_t nblocks = rows * (K / 32);
  const int64_t halves = (int64_t)gridDim.x * (blockDim.x / 16);
  for (int64_t b0 = blockIdx.x * (int64_t)(blockDim.x / 16) + (threadIdx.x & ~31) / 16;
       b0 < nblocks + 1; b0 += halves) {
    // both halves of a warp stay in the loop together (shuffles below)
    const int64_t b = b0 + ((threadIdx.x >> 4) & 1);
    const bool live = b < nblocks;
    float2 v = make_float2(0.f, 0.f);
    if (live) v = __ldg(reinterpret_cast<const float2*>(w + b * 32) + lane);
    float m = fmaxf(fabsf(v.x), fabsf(v.y));
#pragma unroll
    for (int o = 8; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (b0 >= nblocks) break;  // uniform across the warp
    if (!live) continue;
    uint32_t c0 = 0, c1 = 0, sbyte = 0;
    if (m > 0.0f) {
      int e2;
      (void)frexpf(m, &e2);  // m = f * 2^e2, f in [0.5, 1)
      int X = (e2 - 1) - 2;  // floor(log2 m) - 2
      X = X < -127 ? -127 : (X > 127 ? 127 : X);
      sbyte = (uint32_t)(X + 127);
      const float s0 = ldexpf(v.x, -X), s1 = ldexpf(v.y, -X);
      c0 = e2m1_nearest(fabsf(s0)) | (signbit(s0) ? 8u : 0u);
      c1 = e2m1_nearest(fabsf(s1)) | (signbit(s1) ? 8u : 0u);
    }
    blocks[b * 16 + lane] = (uint8_t)(c0 | (c1 << 4));  // even k: low nibble
    if (lane == 0) scales[b] = (uint8_t)sbyte;
  }
}

int grid_for(int64_t work, int threads) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  int64_t blocks = (work + threads - 1) / threads;
  int64_t cap = (int64_t)sms * 8;  // 8 resident 256-thread blocks per SM
  if (blocks > cap) blocks = cap;
  return (int)(blocks < 1 ? 1 : blocks);
}

}  // namespace

cudaError_t launch_dequant(Fmt f, const uint8_t* w, const void* scale,
                           int64_t rows, int64_t K, uint16_t* out,
                           cudaStream_t s) {
  if (rows == 0 || K == 0) return cudaSuccess;
  const int64_t work = rows * (K / 32);
  const int g = grid_for(work, 256);
  if (f == Fmt::NF4)
    nf4_dequant_kernel<<<g, 256, 0, s>>>(w, (const float*)scale, rows, K, out);
  else
    mxfp4_dequant_kernel<<<g, 256, 0, s>>>(w, (const uint8_t*)scale, rows, K,
                                           out);
  return cudaGetLastError();
}

cudaError_t launch_quantize(Fmt f, const float* w, int64_t rows, int64_t K,
                            uint8_t* codes, void* scale, cudaStream_t s) {
  if (rows == 0 || K == 0) return cudaSuccess;
  if (f == Fmt::NF4) {
    const int g = grid_for(rows * (K / 64) * 32, 256);
    nf4_quantize_kernel<<<g, 256, 0, s>>>(w, rows, K, codes, (float*)scale);
  } else {
    const int g = grid_for(rows * (K / 32) * 16, 256);
    mxfp4_quantize_kernel<<<g, 256, 0, s>>>(w, rows, K, codes,
                                            (uint8_t*)scale);
  }
  return cudaGetLastError();
}

}  // namespace gbw
