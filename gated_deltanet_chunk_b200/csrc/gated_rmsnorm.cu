// gated_rmsnorm.cu -- the gated RMSNorm epilogue as its own kernel.
//
// RMSNormGated of the "手撕Qwen3-Next" walkthrough (sections 一(一)1 and 6,
// with the RMSNorm code of section 三): for every row of `dim` values
//
//   y = o / sqrt(mean(o^2) + eps) * w * silu(z)
//
// The decode kernel fuses this into its output store; the chunked forward runs
// this kernel in place on its output, and gdn_gated_rmsnorm exposes it alone.
// It is bound by HBM: per row it reads o and z and writes y once.  Each thread
// moves 16-byte vectors of o, z and y; a row spans dim * esz / 16 lanes
// (8 or 16 for bf16, 16 or 32 for fp32), reduced with shuffles inside its lane
// group.  A grid-stride loop over passes of U rows per lane group keeps the
// grid at a multiple of the SM count.
#include "gdn_common.cuh"
#include "gdn_silu.cuh"
#include "gdn_launch.h"

namespace gdn {
namespace rmsnorm {

constexpr int kThreads = 256;

// 16-byte vectors: loaded as raw words, unpacked to fp32 only when used.
template <typename IO> struct Vec;
template <> struct Vec<float> {
  static constexpr int N = 4;
  __device__ static uint4 load(const void* p) { return __ldcs(reinterpret_cast<const uint4*>(p)); }
  __device__ static void unpack(uint4 v, float* x) {
    x[0] = __uint_as_float(v.x); x[1] = __uint_as_float(v.y);
    x[2] = __uint_as_float(v.z); x[3] = __uint_as_float(v.w);
  }
  __device__ static void store(void* p, const float* x) {
    __stcs(reinterpret_cast<float4*>(p), make_float4(x[0], x[1], x[2], x[3]));
  }
};
template <> struct Vec<__nv_bfloat16> {
  static constexpr int N = 8;
  __device__ static uint4 load(const void* p) { return __ldcs(reinterpret_cast<const uint4*>(p)); }
  __device__ static void unpack(uint4 v, float* x) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      x[2 * i] = __uint_as_float(w[i] << 16);
      x[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
  }
  __device__ static void store(void* p, const float* x) {
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const __nv_bfloat162 h = __floats2bfloat162_rn(x[2 * i], x[2 * i + 1]);
      w[i] = *reinterpret_cast<const uint32_t*>(&h);
    }
    __stcs(reinterpret_cast<uint4*>(p), make_uint4(w[0], w[1], w[2], w[3]));
  }
};

// U rows per lane group per pass: all 2U vector loads are issued before any
// of them is used, so each thread keeps 32U bytes in flight.
constexpr int U = 4;

template <typename IO, int DIM>
__global__ void __launch_bounds__(kThreads) gated_rmsnorm_kernel(const IO* __restrict__ o, const IO* __restrict__ z,
                                                                 const float* __restrict__ w, float eps,
                                                                 IO* y, int64_t rows) {
  constexpr int E = Vec<IO>::N;     // elements per thread
  constexpr int L = DIM / E;        // lanes per row
  constexpr int G = kThreads / L;   // lane groups per block
  static_assert(L <= 32 && 32 % L == 0, "row must fit a warp");
  const int lane_in_row = threadIdx.x % L;
  float wv[E];
#pragma unroll
  for (int e = 0; e < E; ++e) wv[e] = w[lane_in_row * E + e];
  // pass p covers rows [p * G * U, (p + 1) * G * U); group g takes rows g, g + G, ... of it
  const int64_t passes = (rows + (int64_t)G * U - 1) / ((int64_t)G * U);
  for (int64_t pidx = blockIdx.x; pidx < passes; pidx += gridDim.x) {
    const int64_t r0 = pidx * G * U + threadIdx.x / L;
    uint4 ow[U], zw[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int64_t r = r0 + (int64_t)u * G;
      const size_t off = (size_t)r * DIM + lane_in_row * E;
      ow[u] = r < rows ? Vec<IO>::load(o + off) : make_uint4(0u, 0u, 0u, 0u);
      zw[u] = r < rows ? Vec<IO>::load(z + off) : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int64_t r = r0 + (int64_t)u * G;
      float ov[E], zv[E];
      Vec<IO>::unpack(ow[u], ov);
      float ss = 0.f;
#pragma unroll
      for (int e = 0; e < E; ++e) ss = fmaf(ov[e], ov[e], ss);
#pragma unroll
      for (int m = L / 2; m > 0; m >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, m);
      if (r < rows) {
        Vec<IO>::unpack(zw[u], zv);
        const float inv = rsqrtf(ss * (1.f / DIM) + eps);
#pragma unroll
        for (int e = 0; e < E; ++e) ov[e] = ov[e] * inv * wv[e] * silu_io<IO>(zv[e]);
        Vec<IO>::store(y + (size_t)r * DIM + lane_in_row * E, ov);
      }
    }
  }
}

template <typename IO, int DIM>
static cudaError_t launch_one(const void* o, const void* z, const float* w, float eps, void* y, int64_t rows,
                              cudaStream_t s) {
  constexpr int RPB = kThreads / (DIM / Vec<IO>::N) * U;  // rows per block per pass
  int dev = 0, sms = 148, per_sm = 1;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, gated_rmsnorm_kernel<IO, DIM>, kThreads, 0);
  const int64_t need = (rows + RPB - 1) / RPB;
  const int64_t cap = (int64_t)sms * (per_sm > 0 ? per_sm : 1);  // one wave of resident blocks
  const int grid = (int)(need < cap ? need : cap);
  gated_rmsnorm_kernel<IO, DIM><<<grid, kThreads, 0, s>>>(static_cast<const IO*>(o), static_cast<const IO*>(z),
                                                          w, eps, static_cast<IO*>(y), rows);
  return cudaGetLastError();
}

}  // namespace rmsnorm

cudaError_t launch_gated_rmsnorm(const void* o, const void* z, const float* w, float eps, void* y, int64_t rows,
                                 int dim, int io_bf16, cudaStream_t s) {
  using bf = __nv_bfloat16;
  if (rows == 0) return cudaSuccess;
  if (dim == 64) return io_bf16 ? rmsnorm::launch_one<bf, 64>(o, z, w, eps, y, rows, s)
                                : rmsnorm::launch_one<float, 64>(o, z, w, eps, y, rows, s);
  if (dim == 128) return io_bf16 ? rmsnorm::launch_one<bf, 128>(o, z, w, eps, y, rows, s)
                                 : rmsnorm::launch_one<float, 128>(o, z, w, eps, y, rows, s);
  return cudaErrorInvalidValue;
}

}  // namespace gdn
