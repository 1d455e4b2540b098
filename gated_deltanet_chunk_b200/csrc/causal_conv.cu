// causal_conv.cu -- causal depthwise conv1d + SiLU of the packed q|k|v channels.
//
// The "手撕Qwen3-Next" walkthrough, section 一(一)3 (qkv 卷积部分): every channel
// of mixed_qkv = [q | k | v] is convolved on its own with K taps, zero padded by
// K - 1 on the left and cut to the sequence (a causal cross-correlation), then
// passed through SiLU:
//
//   y[t, c] = silu(bias[c] + sum_i w[c, i] * in(t - (K - 1) + i))
//
// where in(p) is the input at position p of the sequence, or, for p < 0, the
// cached window before it (conv_state[n, c, K + p]; zeros without one).  The
// decode update (torch_causal_conv1d_update) is the same formula over
// [conv_state, x] for one token, and the new conv_state is the last K inputs.
//
// The outputs go straight to the three tensors the chunk and decode kernels
// read: channels [0, Nqk Dk) to q [T, Nqk, Dk], [Nqk Dk, 2 Nqk Dk) to k, the
// rest to v [T, Nv, Dv].  Every kernel here is bound by HBM: x is read once
// and q, k, v written once (a prefill block also reads the K - 1 rows before
// its first token, 3 in 128, which the neighbouring block has brought into
// L2).  A thread owns one 16-byte vector of channels (8 bf16 or 4 fp32).
#include "gdn_common.cuh"
#include "gdn_silu.cuh"
#include "gdn_launch.h"

namespace gdn {
namespace conv {

constexpr int kThreads = 256;
constexpr int kTokensPerBlock = 128;  // prefill: consecutive tokens per thread (64 and 32 measured slower)

template <typename IO> struct V16;
template <> struct V16<float> {
  static constexpr int N = 4;
  __device__ static void store(void* p, const float* x) {
    *reinterpret_cast<float4*>(p) = make_float4(x[0], x[1], x[2], x[3]);
  }
};
template <> struct V16<__nv_bfloat16> {
  static constexpr int N = 8;
  __device__ static void store(void* p, const float* x) {
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const __nv_bfloat162 h = __floats2bfloat162_rn(x[2 * i], x[2 * i + 1]);
      w[i] = *reinterpret_cast<const uint32_t*>(&h);
    }
    *reinterpret_cast<uint4*>(p) = make_uint4(w[0], w[1], w[2], w[3]);
  }
};

// Raw 16-byte vectors, unpacked to fp32 when used.
__device__ __forceinline__ uint4 ld16(const void* p) { return *reinterpret_cast<const uint4*>(p); }
template <typename IO> __device__ __forceinline__ void unpack16(uint4 v, float* x);
template <> __device__ __forceinline__ void unpack16<float>(uint4 v, float* x) {
  x[0] = __uint_as_float(v.x); x[1] = __uint_as_float(v.y); x[2] = __uint_as_float(v.z); x[3] = __uint_as_float(v.w);
}
template <> __device__ __forceinline__ void unpack16<__nv_bfloat16>(uint4 v, float* x) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    x[2 * i] = __uint_as_float(w[i] << 16);
    x[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}

// The taps and bias of channels [c0, c0 + E): w[i][e], b[e] (16-byte loads; the
// E * K weights of a thread are contiguous and 16-byte aligned).
template <int E, int K>
__device__ __forceinline__ void load_taps(const ConvArgs& a, int c0, float (&w)[K][E], float (&b)[E]) {
  const float4* wp = reinterpret_cast<const float4*>(a.weight + (size_t)c0 * K);
#pragma unroll
  for (int q = 0; q < E * K / 4; ++q) {
    const float4 v = __ldg(wp + q);
    const float f[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int r = 0; r < 4; ++r) w[(4 * q + r) % K][(4 * q + r) / K] = f[r];
  }
#pragma unroll
  for (int e = 0; e < E; ++e) b[e] = a.bias ? __ldg(a.bias + c0 + e) : 0.f;
}

// Destination of channel vector c0 (E channels starting at c0) for row t.
template <typename IO>
__device__ __forceinline__ IO* out_ptr(const ConvArgs& a, int64_t t, int c0) {
  const int qk = a.nqk * a.dk;
  if (c0 < qk) return static_cast<IO*>(a.q) + (size_t)t * qk + c0;
  if (c0 < 2 * qk) return static_cast<IO*>(a.k) + (size_t)t * qk + (c0 - qk);
  const int vd = a.nv * a.dv;
  return static_cast<IO*>(a.v) + (size_t)t * vd + (c0 - 2 * qk);
}

// Channel c of the window before sequence n: conv_state[row, c, j], j in [0, K).
template <typename IO>
__device__ __forceinline__ float window_at(const ConvArgs& a, int64_t row, int c, int j) {
  if (a.state_in == nullptr || row < 0 || j < 0 || j >= a.ksize) return 0.f;
  return to_f32(static_cast<const IO*>(a.state_in)[((size_t)row * a.channels + c) * a.ksize + j]);
}

// Sequence of token t (cu is non-decreasing; the first n with cu[n+1] > t).
__device__ __forceinline__ int seq_of(const int32_t* cu, int num_seqs, int64_t t) {
  int lo = 0, hi = num_seqs - 1;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if ((int64_t)cu[mid + 1] > t) hi = mid; else lo = mid + 1;
  }
  return lo;
}

// Prefill: block (token block, channel block); thread = one channel vector over
// kTokensPerBlock consecutive tokens, which may cross sequence boundaries.  The
// thread's input rows come through a ring of kDepth 16-byte cp.async copies in
// shared memory, so kDepth - 1 rows stay in flight without holding registers.
// A thread reads back only the slots it filled itself, so its own
// cp.async.wait_group orders them and no block barrier is needed.  The K - 1
// previous inputs stay in registers as a sliding window, and the token loop is
// unrolled by 4 so that shifting it costs no moves.  On the long prefill
// (65,536 tokens x 8192 channels, bf16) the steps measured: register-held
// double buffer of 4 rows 0.494 ms; with the one-MUFU SiLU 0.406 ms; this ring
// 0.381 ms; unrolled 0.358 ms.  Deeper rings (24) and three blocks per SM
// (register spills) measured slower.
constexpr int kDepth = 16;
constexpr int kBlocksPerSM = 2;

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

template <typename IO, int K>
__global__ void __launch_bounds__(kThreads, kBlocksPerSM) conv_fwd_kernel(ConvArgs a) {
  constexpr int E = V16<IO>::N;
  extern __shared__ __align__(16) uint4 ring[];  // [kDepth][kThreads]
  const int c0 = (blockIdx.y * kThreads + threadIdx.x) * E;
  if (c0 >= a.channels) return;
  const int64_t t_begin = (int64_t)blockIdx.x * kTokensPerBlock;
  const int64_t t_end = min((int64_t)a.total_tokens, t_begin + kTokensPerBlock);
  if (t_begin >= t_end) return;
  const IO* xc = static_cast<const IO*>(a.x) + c0;
  const uint32_t rbase = (uint32_t)__cvta_generic_to_shared(ring + threadIdx.x);
  // row tt into ring slot `slot`; one commit group per row (empty past the block's rows)
  auto fetch = [&](int64_t tt, int slot) {
    if (tt < t_end) cp_async16(rbase + (uint32_t)(slot * kThreads * 16), xc + (size_t)tt * a.channels);
    cp_async_commit();
  };
#pragma unroll
  for (int u = 0; u + 1 < kDepth; ++u) fetch(t_begin + u, u);
  float w[K][E], b[E];
  load_taps<E, K>(a, c0, w, b);
  int n = a.cu ? seq_of(a.cu, a.num_seqs, t_begin) : (int)(t_begin / a.uniform_len);
  int64_t s_begin, s_end;
  seq_bounds(a, n, s_begin, s_end);
  // win[j] = input at position t - (K - 1) + j for the next token t
  float win[K > 1 ? K - 1 : 1][E];
#pragma unroll
  for (int j = 0; j + 1 < K; ++j) {
    const int64_t p = t_begin - (K - 1) + j;
    if (p >= s_begin) {
      unpack16<IO>(ld16(xc + (size_t)p * a.channels), win[j]);
    } else {
#pragma unroll
      for (int e = 0; e < E; ++e) win[j][e] = window_at<IO>(a, n, c0 + e, (int)(K + (p - s_begin)));
    }
  }
  const int rows = (int)(t_end - t_begin);
#pragma unroll 4  // the window shifts become register renames
  for (int i = 0; i < rows; ++i) {
    const int64_t t = t_begin + i;
    // refill the slot read in the previous iteration, then wait for row i
    fetch(t + kDepth - 1, (i + kDepth - 1) % kDepth);
    cp_async_wait<kDepth - 1>();
    const uint4 raw = ring[(i % kDepth) * kThreads + threadIdx.x];
    if (t >= s_end) {  // first token of the next non-empty sequence: restart the window
      while (t >= s_end && n + 1 < a.num_seqs) {
        ++n;
        seq_bounds(a, n, s_begin, s_end);
      }
#pragma unroll
      for (int j = 0; j + 1 < K; ++j)
#pragma unroll
        for (int e = 0; e < E; ++e) win[j][e] = window_at<IO>(a, n, c0 + e, j + 1);
    }
    // a token of no sequence (only with inconsistent cu_seqlens, already reported) is not stored
    const bool outside = t < s_begin || t >= s_end;
    float xt[E], acc[E];
    unpack16<IO>(raw, xt);
#pragma unroll
    for (int e = 0; e < E; ++e) {
      float s_ = b[e];
#pragma unroll
      for (int j = 0; j + 1 < K; ++j) s_ = fmaf(w[j][e], win[j][e], s_);
      acc[e] = silu_io<IO>(fmaf(w[K - 1][e], xt[e], s_));
    }
    if (!outside) V16<IO>::store(out_ptr<IO>(a, t, c0), acc);
#pragma unroll
    for (int j = 0; j + 2 < K; ++j)
#pragma unroll
      for (int e = 0; e < E; ++e) win[j][e] = win[j + 1][e];
    if (K > 1) {
#pragma unroll
      for (int e = 0; e < E; ++e) win[K > 1 ? K - 2 : 0][e] = xt[e];
    }
  }
  cp_async_wait<0>();  // no copy outlives the block
}

// The conv_state after a prefill: the last K inputs of [window, sequence] of
// every sequence (thread = one channel of one sequence).  Runs after
// conv_fwd_kernel on the same stream, so state_out may be state_in.
template <typename IO, int K>
__global__ void __launch_bounds__(kThreads) conv_state_kernel(ConvArgs a) {
  const int64_t idx = (int64_t)blockIdx.x * kThreads + threadIdx.x;
  if (idx >= (int64_t)a.num_seqs * a.channels) return;
  const int n = (int)(idx / a.channels), c = (int)(idx % a.channels);
  int64_t s_begin, s_end;
  seq_bounds(a, n, s_begin, s_end);
  const int64_t len = s_end - s_begin;
  float v[K];
#pragma unroll
  for (int i = 0; i < K; ++i) {
    const int64_t p = len - K + i;  // position in the sequence
    v[i] = p >= 0 ? to_f32(static_cast<const IO*>(a.x)[(size_t)(s_begin + p) * a.channels + c])
                  : window_at<IO>(a, n, c, (int)(K + p));
  }
  IO* dst = static_cast<IO*>(a.state_out) + ((size_t)n * a.channels + c) * K;
#pragma unroll
  for (int i = 0; i < K; ++i) dst[i] = from_f32<IO>(v[i]);
}

// Decode: one token per sequence, conv_state updated in place (optionally
// through slot ids).  Thread = one channel vector of one sequence; its state
// span (E channels x K taps, 16 K bytes) and its taps move as 16-byte vectors.
template <typename IO, int K>
__global__ void __launch_bounds__(kThreads) conv_update_kernel(ConvArgs a) {
  constexpr int E = V16<IO>::N;
  constexpr int PER = 16 / (int)sizeof(IO);  // state elements per 16-byte vector
  const int c0 = (blockIdx.x * kThreads + threadIdx.x) * E;
  const int n = blockIdx.y;
  if (c0 >= a.channels) return;
  int64_t row = n;
  if (a.slots) {
    const int32_t s = a.slots[n];
    row = (s >= 0 && s < a.num_slots) ? s : -1;
  }
  float out[E];
  if (row < 0) {  // a padding sequence: zero output, no state
#pragma unroll
    for (int e = 0; e < E; ++e) out[e] = 0.f;
    V16<IO>::store(out_ptr<IO>(a, n, c0), out);
    return;
  }
  const uint4 xr = ld16(static_cast<const IO*>(a.x) + (size_t)n * a.channels + c0);
  IO* st = static_cast<IO*>(a.state_out) + ((size_t)row * a.channels + c0) * K;
  uint4 sr[K];  // E * K state elements, channel-major: element (e, i) at e * K + i
#pragma unroll
  for (int q = 0; q < K; ++q) sr[q] = ld16(st + q * PER);
  float w[K][E], b[E];
  load_taps<E, K>(a, c0, w, b);
  float x[E], win[E * K];
  unpack16<IO>(xr, x);
#pragma unroll
  for (int q = 0; q < K; ++q) unpack16<IO>(sr[q], win + q * PER);
#pragma unroll
  for (int e = 0; e < E; ++e) {
    // taps 0..K-2 meet the window's entries 1..K-1, tap K-1 the new input
    float acc = b[e];
#pragma unroll
    for (int i = 0; i + 1 < K; ++i) acc = fmaf(w[i][e], win[e * K + i + 1], acc);
    out[e] = silu_io<IO>(fmaf(w[K - 1][e], x[e], acc));
  }
  // the new window: shifted by one, the new input last
#pragma unroll
  for (int e = 0; e < E; ++e) {
#pragma unroll
    for (int i = 0; i + 1 < K; ++i) win[e * K + i] = win[e * K + i + 1];
    win[e * K + K - 1] = x[e];
  }
#pragma unroll
  for (int q = 0; q < K; ++q) V16<IO>::store(st + q * PER, win + q * PER);
  V16<IO>::store(out_ptr<IO>(a, n, c0), out);
}

// Decode update for K in {1, 2, 4}: a thread owns CH channels of kSeqPerThread
// sequences, CH chosen so that its state span (CH channels x K taps) is one
// 16-byte vector.  A warp's state loads and stores are then contiguous 512-byte
// runs and its x / q, k, v accesses contiguous too, and the thread's taps (CH K
// fp32: one or two 16-byte vectors) are loaded once for all its sequences.  The
// kernel above spans 16 K bytes of state and 4 K floats of taps per thread, so a
// warp-wide access touches 16 to 32 cache lines: its L1 data pipe, not DRAM,
// set the pace (87 % busy, DRAM 12 %).  All sequences' loads are issued before
// any is used.  The decode workload's update (256 sequences, 8192 channels,
// 42 MB) measured 18.8 us with that kernel and 8.6 us with this one (2
// sequences per thread; 4: 8.75 us, 8: 9.8 us), CUDA graphs on one box.
constexpr int kSeqPerThread = 2;

template <int B> __device__ __forceinline__ void ld_words(const void* p, uint32_t (&w)[B / 4]) {
  if constexpr (B == 4) {
    w[0] = *reinterpret_cast<const uint32_t*>(p);
  } else if constexpr (B == 8) {
    const uint2 v = *reinterpret_cast<const uint2*>(p);
    w[0] = v.x; w[1] = v.y;
  } else {
    const uint4 v = *reinterpret_cast<const uint4*>(p);
    w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
  }
}
template <int B> __device__ __forceinline__ void st_words(void* p, const uint32_t (&w)[B / 4]) {
  if constexpr (B == 4) {
    *reinterpret_cast<uint32_t*>(p) = w[0];
  } else if constexpr (B == 8) {
    *reinterpret_cast<uint2*>(p) = make_uint2(w[0], w[1]);
  } else {
    *reinterpret_cast<uint4*>(p) = make_uint4(w[0], w[1], w[2], w[3]);
  }
}
// W 32-bit words <-> the 4 W / sizeof(IO) values of IO they hold (low half first)
template <typename IO, int W> __device__ __forceinline__ void unpack_words(const uint32_t (&w)[W], float* x) {
  if constexpr (sizeof(IO) == 4) {
#pragma unroll
    for (int i = 0; i < W; ++i) x[i] = __uint_as_float(w[i]);
  } else {
#pragma unroll
    for (int i = 0; i < W; ++i) {
      x[2 * i] = __uint_as_float(w[i] << 16);
      x[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
  }
}
template <typename IO, int W> __device__ __forceinline__ void pack_words(const float* x, uint32_t (&w)[W]) {
  if constexpr (sizeof(IO) == 4) {
#pragma unroll
    for (int i = 0; i < W; ++i) w[i] = __float_as_uint(x[i]);
  } else {
#pragma unroll
    for (int i = 0; i < W; ++i) {
      const __nv_bfloat162 h = __floats2bfloat162_rn(x[2 * i], x[2 * i + 1]);
      w[i] = *reinterpret_cast<const uint32_t*>(&h);
    }
  }
}

template <typename IO, int K>
__global__ void __launch_bounds__(kThreads) conv_update_packed_kernel(ConvArgs a) {
  static_assert(K == 1 || K == 2 || K == 4, "the state span of CH channels is one 16-byte vector");
  constexpr int ESZ = (int)sizeof(IO);
  constexpr int CH = 16 / (K * ESZ);  // channels per thread
  constexpr int XB = CH * ESZ;        // bytes of x and of the output per thread: 4, 8 or 16
  const int c0 = (blockIdx.x * kThreads + threadIdx.x) * CH;
  if (c0 >= a.channels) return;
  float w[CH][K], b[CH];
  {
    const float4* wp = reinterpret_cast<const float4*>(a.weight + (size_t)c0 * K);  // CH K = 16 / ESZ floats
#pragma unroll
    for (int q = 0; q < CH * K / 4; ++q) {
      const float4 v = __ldg(wp + q);
      const float f[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int r = 0; r < 4; ++r) w[(4 * q + r) / K][(4 * q + r) % K] = f[r];
    }
#pragma unroll
    for (int e = 0; e < CH; ++e) b[e] = a.bias ? __ldg(a.bias + c0 + e) : 0.f;
  }
  const int n0 = blockIdx.y * kSeqPerThread;
  int64_t rows[kSeqPerThread];  // state row; -1 for a padding sequence, -2 past the batch
  uint32_t xw[kSeqPerThread][XB / 4];
  uint4 sw[kSeqPerThread];
#pragma unroll
  for (int s = 0; s < kSeqPerThread; ++s) {
    const int n = n0 + s;
    int64_t row = -2;
    if (n < a.num_seqs) {
      row = n;
      if (a.slots) {
        const int32_t id = a.slots[n];
        row = (id >= 0 && id < a.num_slots) ? id : -1;
      }
    }
    rows[s] = row;
    if (row >= 0) {
      ld_words<XB>(static_cast<const IO*>(a.x) + (size_t)n * a.channels + c0, xw[s]);
      sw[s] = ld16(static_cast<const IO*>(a.state_out) + ((size_t)row * a.channels + c0) * K);
    }
  }
#pragma unroll
  for (int s = 0; s < kSeqPerThread; ++s) {
    const int n = n0 + s;
    if (rows[s] == -2) break;
    float out[CH];
    if (rows[s] >= 0) {
      float x[CH], win[CH * K];  // window: channel e's entries at e K .. e K + K - 1, oldest first
      unpack_words<IO, XB / 4>(xw[s], x);
      unpack16<IO>(sw[s], win);
#pragma unroll
      for (int e = 0; e < CH; ++e) {
        // taps 0..K-2 meet the window's entries 1..K-1, tap K-1 the new input
        float acc = b[e];
#pragma unroll
        for (int i = 0; i + 1 < K; ++i) acc = fmaf(w[e][i], win[e * K + i + 1], acc);
        out[e] = silu_io<IO>(fmaf(w[e][K - 1], x[e], acc));
#pragma unroll
        for (int i = 0; i + 1 < K; ++i) win[e * K + i] = win[e * K + i + 1];
        win[e * K + K - 1] = x[e];
      }
      V16<IO>::store(static_cast<IO*>(a.state_out) + ((size_t)rows[s] * a.channels + c0) * K, win);
    } else {
#pragma unroll
      for (int e = 0; e < CH; ++e) out[e] = 0.f;  // a padding sequence: zero output, no state
    }
    uint32_t ow[XB / 4];
    pack_words<IO, XB / 4>(out, ow);
    st_words<XB>(out_ptr<IO>(a, n, c0), ow);
  }
}

template <typename IO, int K>
static cudaError_t launch_fwd(const ConvArgs& a, cudaStream_t s) {
  constexpr int E = V16<IO>::N;
  const int vecs = a.channels / E;
  if (a.total_tokens > 0) {
    dim3 grid((unsigned)((a.total_tokens + kTokensPerBlock - 1) / kTokensPerBlock), (vecs + kThreads - 1) / kThreads);
    constexpr size_t smem = (size_t)kDepth * kThreads * 16;
    cudaError_t e = cudaFuncSetAttribute(conv_fwd_kernel<IO, K>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    conv_fwd_kernel<IO, K><<<grid, kThreads, smem, s>>>(a);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  if (a.state_out) {
    const int64_t thr = (int64_t)a.num_seqs * a.channels;
    conv_state_kernel<IO, K><<<(unsigned)((thr + kThreads - 1) / kThreads), kThreads, 0, s>>>(a);
  }
  return cudaGetLastError();
}

template <typename IO, int K>
static cudaError_t launch_update(const ConvArgs& a, cudaStream_t s) {
  if constexpr (K == 3) {  // 3 taps x any channel count is no 16-byte span: a channel vector per thread
    constexpr int E = V16<IO>::N;
    dim3 grid((a.channels / E + kThreads - 1) / kThreads, a.num_seqs);
    conv_update_kernel<IO, K><<<grid, kThreads, 0, s>>>(a);
  } else {
    constexpr int CH = 16 / (K * (int)sizeof(IO));
    dim3 grid((a.channels / CH + kThreads - 1) / kThreads, (a.num_seqs + kSeqPerThread - 1) / kSeqPerThread);
    conv_update_packed_kernel<IO, K><<<grid, kThreads, 0, s>>>(a);
  }
  return cudaGetLastError();
}

template <typename IO>
static cudaError_t dispatch(const ConvArgs& a, bool update, cudaStream_t s) {
  switch (a.ksize) {
    case 1: return update ? launch_update<IO, 1>(a, s) : launch_fwd<IO, 1>(a, s);
    case 2: return update ? launch_update<IO, 2>(a, s) : launch_fwd<IO, 2>(a, s);
    case 3: return update ? launch_update<IO, 3>(a, s) : launch_fwd<IO, 3>(a, s);
    case 4: return update ? launch_update<IO, 4>(a, s) : launch_fwd<IO, 4>(a, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace conv

cudaError_t launch_conv_fwd(const ConvArgs& a, int io_bf16, cudaStream_t s) {
  return io_bf16 ? conv::dispatch<__nv_bfloat16>(a, false, s) : conv::dispatch<float>(a, false, s);
}

cudaError_t launch_conv_update(const ConvArgs& a, int io_bf16, cudaStream_t s) {
  return io_bf16 ? conv::dispatch<__nv_bfloat16>(a, true, s) : conv::dispatch<float>(a, true, s);
}

}  // namespace gdn
