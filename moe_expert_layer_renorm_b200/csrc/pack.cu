// NVFP4 pack of an fp32 tensor [N, K]: per-tensor fp32 scale, one E4M3 scale
// per 16 consecutive K of a row, two E2M1 codes per byte (even k low nibble).
// Every step is an IEEE fp32 operation rounded to nearest (no fast math):
//   g   = amax / 2688 (1 if amax == 0)
//   s_b = e4m3_rn_satfinite(amax_b / (6 g))
//   q   = e2m1_rn_satfinite(w / (e4m3(s_b) g)),  0 where e4m3(s_b) == 0
// The conversions to E4M3/E2M1 use the hardware cvt (round to nearest even,
// saturate to the largest finite value).
#include <cuda_fp16.h>
#include "sm100.cuh"

namespace ftmoe {

// Where a packed tensor's bytes go.  Code byte j of row n (codes of k = 2j,
// 2j + 1) lives at codes + (j / 128) * c_stage + n * c_row + j % 128 and
// scale byte b at scales + (b / 16) * s_stage + n * s_row + b % 16: row-major
// [N, K/2] and [N, ld] with (c_row, c_stage, s_row, s_stage) = (K/2, 128,
// ld, 16); stage-tiled [S][N][128] and [S][N][16] with (128, 128 N, 16, 16 N).
// A tiled tensor also gets zero code bytes past K/2 in its last stage.
struct PackPlace {
  uint8_t* codes;
  uint8_t* scales;
  int tiled;
  long long c_row, c_stage, s_row, s_stage;
  __host__ __device__ uint8_t* code_at(int n, long long j) const {
    return codes + (j / 128) * c_stage + n * c_row + (j % 128);
  }
  __host__ __device__ uint8_t* scale_at(int n, long long b) const {
    return scales + (b / 16) * s_stage + n * s_row + (b % 16);
  }
};

static PackPlace row_major_place(uint8_t* codes, uint8_t* scales, int K, int ld_scale) {
  PackPlace p;
  p.codes = codes;
  p.scales = scales;
  p.tiled = 0;
  p.c_row = K / 2;
  p.c_stage = 128;
  p.s_row = ld_scale;
  p.s_stage = 16;
  return p;
}

__global__ void __launch_bounds__(256) amax_kernel(const float4* __restrict__ w, long long n4,
                                                   unsigned int* __restrict__ amax_bits) {
  float m = 0.0f;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n4;
       i += (long long)gridDim.x * blockDim.x) {
    const float4 v = __ldg(w + i);
    m = fmaxf(m, fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, off));
  if ((threadIdx.x & 31) == 0) atomicMax(amax_bits, __float_as_uint(m));  // m >= 0: bits order like values
}

__device__ __forceinline__ uint32_t cvt_e4m3_satfinite(float r) {  // r >= 0
  uint16_t pair;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(pair) : "f"(0.0f), "f"(r));
  return pair & 0xFFu;  // second source lands in the low byte
}

__device__ __forceinline__ float e4m3_to_f32(uint32_t byte) {
  uint32_t h2;
  const uint16_t in = uint16_t(byte);
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(in));
  return __half2float(__ushort_as_half(uint16_t(h2 & 0xFFFFu)));
}

// two fp32 -> one byte of two E2M1 codes: `lo` in bits 3..0, `hi` in bits 7..4
__device__ __forceinline__ uint32_t cvt_e2m1x2_satfinite(float lo, float hi) {
  uint32_t out;
  asm("{.reg .b8 b;\n cvt.rn.satfinite.e2m1x2.f32 b, %1, %2;\n cvt.u32.u8 %0, b;\n}"
      : "=r"(out) : "f"(hi), "f"(lo));
  return out & 0xFFu;
}

// One thread per 16-element block.
__global__ void __launch_bounds__(256) pack_kernel(const float* __restrict__ w, int N, int K, const PackPlace pl,
                                                   int ld_scale, const unsigned int* __restrict__ amax_bits,
                                                   float* __restrict__ global_scale) {
  const int nb = K / 16;
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const float amax = __uint_as_float(*amax_bits);
  const float g = amax > 0.0f ? __fdiv_rn(amax, 2688.0f) : 1.0f;
  if (i == 0) *global_scale = g;
  if (i >= (long long)N * ld_scale) return;
  const int n = int(i / ld_scale), b = int(i % ld_scale);
  if (b >= nb) {  // scale-row padding (and, tiled, the code bytes of the same K range)
    *pl.scale_at(n, b) = 0;
    if (pl.tiled) *reinterpret_cast<uint2*>(pl.code_at(n, 8LL * b)) = make_uint2(0u, 0u);
    return;
  }
  const float4* src = reinterpret_cast<const float4*>(w + size_t(n) * K + size_t(b) * 16);
  float v[16];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const float4 f = __ldg(src + q);
    v[4 * q] = f.x; v[4 * q + 1] = f.y; v[4 * q + 2] = f.z; v[4 * q + 3] = f.w;
  }
  float amax_b = 0.0f;
#pragma unroll
  for (int q = 0; q < 16; ++q) amax_b = fmaxf(amax_b, fabsf(v[q]));
  const float denom = __fmul_rn(6.0f, g);
  const uint32_t sbyte = cvt_e4m3_satfinite(__fdiv_rn(amax_b, denom));
  const float sd = e4m3_to_f32(sbyte);
  const float qden = __fmul_rn(sd, g);
  uint32_t words[2] = {0u, 0u};
  if (sd != 0.0f) {
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const uint32_t byte = cvt_e2m1x2_satfinite(__fdiv_rn(v[2 * q], qden), __fdiv_rn(v[2 * q + 1], qden));
      words[q / 4] |= byte << (8 * (q % 4));
    }
  }
  *reinterpret_cast<uint2*>(pl.code_at(n, 8LL * b)) = make_uint2(words[0], words[1]);
  *pl.scale_at(n, b) = uint8_t(sbyte);
}

static cudaError_t launch_pack(const float* w, int N, int K, const PackPlace& pl, int ld_scale,
                               float* global_scale, void* ws, cudaStream_t s) {
  unsigned int* amax = static_cast<unsigned int*>(ws);
  cudaError_t e = cudaMemsetAsync(amax, 0, sizeof(unsigned int), s);
  if (e != cudaSuccess) return e;
  const long long n4 = (long long)N * K / 4;
  const int blocks1 = int(std::min<long long>((n4 + 255) / 256, 148LL * 8));
  {
    ProfileScope prof(FT_KERNEL_PACK, s);
    amax_kernel<<<blocks1, 256, 0, s>>>(reinterpret_cast<const float4*>(w), n4, amax);
  }
  const long long nthreads = (long long)N * ld_scale;
  ProfileScope prof(FT_KERNEL_PACK, s);
  pack_kernel<<<dim3(unsigned((nthreads + 255) / 256)), 256, 0, s>>>(w, N, K, pl, ld_scale, amax, global_scale);
  return cudaGetLastError();
}

// MXFP4 (OCP Microscaling) pack: one E8M0 scale per 32 consecutive K of a
// row, stored twice so that the slot layout matches NVFP4's one byte per 16:
//   x_b = clamp(floor(log2 amax_b) - 2, -127, 127)   (-127 if amax_b = 0)
//   q   = e2m1_rn_satfinite(w / 2^x_b)               (a power-of-two scaling: exact)
// and the tensor's global = 2^t, t = clamp(floor(log2 amax) - 2) - 13, which
// the GEMMs divide out of every dequantised f16 value (so e2m1 * 2^(x_b - t)
// <= 6 * 2^13) and multiply back in fp32.  A block with x_b - t < -23 would
// lose nonzero values to f16 underflow; it records FT_DEV_F16_RANGE.
// One thread per scale byte position: even positions pack their 32-block.
__global__ void __launch_bounds__(256) mxfp4_pack_kernel(const float* __restrict__ w, int N, int K,
                                                         const PackPlace pl, int ld_scale,
                                                         const unsigned int* __restrict__ amax_bits,
                                                         float* __restrict__ global_scale) {
  const int nb16 = K / 16;
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const float amax = __uint_as_float(*amax_bits);
  const int t = amax > 0.0f ? max(-127, min(127, ilogbf(amax) - 2)) - 13 : 0;
  if (i == 0) *global_scale = ldexpf(1.0f, t);
  if (i >= (long long)N * ld_scale) return;
  const int n = int(i / ld_scale), b16 = int(i % ld_scale);
  if (b16 >= nb16) {  // scale-row padding (and, tiled, the code bytes of the same K range)
    *pl.scale_at(n, b16) = 0;
    if (pl.tiled) *reinterpret_cast<uint2*>(pl.code_at(n, 8LL * b16)) = make_uint2(0u, 0u);
    return;
  }
  if (b16 & 1) return;   // written by the even position of the pair
  const int b = b16 / 2;
  const float4* src = reinterpret_cast<const float4*>(w + size_t(n) * K + size_t(b) * 32);
  float v[32];
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    const float4 f = __ldg(src + q);
    v[4 * q] = f.x; v[4 * q + 1] = f.y; v[4 * q + 2] = f.z; v[4 * q + 3] = f.w;
  }
  float amax_b = 0.0f;
#pragma unroll
  for (int q = 0; q < 32; ++q) amax_b = fmaxf(amax_b, fabsf(v[q]));
  const int x = amax_b > 0.0f ? max(-127, min(127, ilogbf(amax_b) - 2)) : -127;
  if (amax_b > 0.0f && x - t < -23) set_device_status(FT_DEV_F16_RANGE);
  uint32_t words[4] = {0u, 0u, 0u, 0u};
#pragma unroll
  for (int q = 0; q < 16; ++q) {
    const uint32_t byte = cvt_e2m1x2_satfinite(ldexpf(v[2 * q], -x), ldexpf(v[2 * q + 1], -x));
    words[q / 4] |= byte << (8 * (q % 4));
  }
  uint2* dst = reinterpret_cast<uint2*>(pl.code_at(n, 16LL * b));   // 16 bytes inside one 128-byte stage row
  dst[0] = make_uint2(words[0], words[1]);
  dst[1] = make_uint2(words[2], words[3]);
  *pl.scale_at(n, 2 * b) = uint8_t(x + 127);
  *pl.scale_at(n, 2 * b + 1) = uint8_t(x + 127);
}

static cudaError_t launch_pack_mxfp4(const float* w, int N, int K, const PackPlace& pl, int ld_scale,
                                     float* global_scale, void* ws, cudaStream_t s) {
  unsigned int* amax = static_cast<unsigned int*>(ws);
  cudaError_t e = cudaMemsetAsync(amax, 0, sizeof(unsigned int), s);
  if (e != cudaSuccess) return e;
  const long long n4 = (long long)N * K / 4;
  const int blocks1 = int(std::min<long long>((n4 + 255) / 256, 148LL * 8));
  {
    ProfileScope prof(FT_KERNEL_PACK, s);
    amax_kernel<<<blocks1, 256, 0, s>>>(reinterpret_cast<const float4*>(w), n4, amax);
  }
  const long long nthreads = (long long)N * ld_scale;
  ProfileScope prof(FT_KERNEL_PACK, s);
  mxfp4_pack_kernel<<<dim3(unsigned((nthreads + 255) / 256)), 256, 0, s>>>(w, N, K, pl, ld_scale, amax,
                                                                             global_scale);
  return cudaGetLastError();
}

}  // namespace ftmoe
