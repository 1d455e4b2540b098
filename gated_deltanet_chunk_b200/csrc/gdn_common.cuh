// gdn_common.cuh -- small device helpers and the argument blocks shared by the
// gated-delta-rule kernels of libgdn.so (sm_100a only).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace gdn {

constexpr float kNormEps = 1e-6f;  // L2 norm eps, inside the square root

// Bits of the device status word that gdn_device_status reads and clears.
constexpr unsigned int kStatusTimeout = 1u;  // a bounded in-kernel wait expired
constexpr unsigned int kStatusSeqlens = 2u;  // cu_seqlens inconsistent with [0, total_tokens]
constexpr unsigned int kStatusGate = 4u;     // a gate g > 0 (or NaN) reached a kernel that needs g <= 0

__device__ __forceinline__ void report_status(unsigned int* status, unsigned int bit) {
  if (status) atomicOr(status, bit);
}

// Arguments of the chunked forward (gdn_chunk_fwd); pointers are device memory.
struct ChunkArgs {
  const void* q;             // [T, Nqk, Dk]
  const void* k;             // [T, Nqk, Dk]
  const void* v;             // [T, Nv, Dv]
  const float* g;            // [T, Nv]: g, or the raw projection a when A_log != nullptr
  const float* beta;         // [T, Nv]: beta, or the raw projection b when A_log != nullptr
  const float* A_log;        // [Nv] or nullptr (g and beta given)
  const float* dt_bias;      // [Nv] (used with A_log)
  const float* s0;           // [N, Nv, Dk, Dv] (or [num_slots, ...] with slots) or nullptr
  const int32_t* slots;      // [N] state row of each sequence, or nullptr (row n)
  int32_t num_slots;         // rows of the state pool when slots != nullptr
  const int32_t* cu;         // [N + 1] or nullptr (equal lengths)
  void* out;                 // [T, Nv, Dv]
  float* s_final;            // [N, Nv, Dk, Dv] or nullptr
  int32_t uniform_len;       // sequence length when cu == nullptr
  int32_t num_seqs;
  int64_t total_tokens;      // T: rows of the token tensors
  unsigned int* status;      // device status word (kStatus* bits)
  int32_t nqk, nv, dv;
  int32_t qk_l2norm;
  float scale;
  const void* nz;            // [T, Nv, Dv] gate of the RMSNorm epilogue, or nullptr (no norm)
  const float* nw;           // [Dv] RMSNorm gain (with nz)
  float neps;                // RMSNorm eps (with nz)
};

// Arguments of the one-token decode step (gdn_recurrent_step).
struct StepArgs {
  const void* q;     // [N, Nqk, Dk]
  const void* k;     // [N, Nqk, Dk]
  const void* v;     // [N, Nv, Dv]
  const float* g;    // [N, Nv]: g, or the raw projection a when A_log != nullptr
  const float* beta; // [N, Nv]: beta, or the raw projection b when A_log != nullptr
  const float* A_log;    // [Nv] or nullptr (g and beta given)
  const float* dt_bias;  // [Nv] (used with A_log)
  float* state;      // [N, Nv, Dk, Dv] (or [num_slots, ...] with slots) in place
  const int32_t* slots;  // [N] state row of each sequence, or nullptr (row n)
  int32_t num_slots;     // rows of the state pool when slots != nullptr
  void* out;         // [N, Nv, Dv]
  int32_t num_seqs;
  int32_t nqk, nv;
  int32_t qk_l2norm;
  float scale;
  const void* nz;      // [N, Nv, Dv] gate of the RMSNorm epilogue, or nullptr (no norm)
  const float* nw;     // [Dv] RMSNorm gain (with nz)
  float neps;          // RMSNorm eps (with nz)
  const void* cx;      // [N, C] packed q|k|v projection when the conv is fused (q, k, v unused), or nullptr
  void* cstate;        // [rows, C, cks] conv state (rows as the recurrent state), updated in place
  const float* cw;     // [C, cks] conv taps
  const float* cb;     // [C] conv bias or nullptr
  int32_t cks;         // conv taps, 1..4
};

// Arguments of the causal conv1d + SiLU of the packed q|k|v channels.
struct ConvArgs {
  const void* x;             // [T, channels] (prefill) or [N, channels] (decode), io dtype
  const float* weight;       // [channels, ksize]
  const float* bias;         // [channels] or nullptr
  const void* state_in;      // [N, channels, ksize] window before each sequence, or nullptr (zeros)
  void* state_out;           // [N, channels, ksize] (prefill: or nullptr); decode: the state, in place
  const int32_t* cu;         // [N + 1] or nullptr (equal lengths)
  const int32_t* slots;      // decode: [N] state row of each sequence, or nullptr (row n)
  int32_t num_slots;
  int32_t uniform_len;       // sequence length when cu == nullptr
  int32_t num_seqs;
  int64_t total_tokens;
  int32_t channels, ksize;   // channels = 2 nqk dk + nv dv
  int32_t nqk, nv, dk, dv;
  unsigned int* status;      // device status word (kStatus* bits)
  void* q;                   // [T or N, nqk, dk] outputs
  void* k;
  void* v;                   // [T or N, nv, dv]
};

template <typename T> __device__ __forceinline__ float to_f32(T x);
template <> __device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) {
  return __bfloat162float(x);
}

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);  // round to nearest even
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

// The gate of row i (a token, or a sequence in a decode step) on v-head h.
// Without A_log the caller passed g and beta.  With it, the g / beta slots hold
// the layer's raw projections a and b, and the gate is formed as in the
// "手撕Qwen3-Next" walkthrough, section 一(一)4:
//   beta = sigmoid(b),  g = -exp(A_log[h]) * softplus(a + dt_bias[h]),
// softplus(x) = log(1 + exp(x)), evaluated as max(x, 0) + log1p(exp(-|x|)).
template <class Args>
__device__ __forceinline__ void gate_from_raw(const Args& a, size_t i, int h, float& g, float& beta) {
  const float u = a.g[i] + a.dt_bias[h];
  g = -expf(a.A_log[h]) * (fmaxf(u, 0.f) + log1pf(expf(-fabsf(u))));
  beta = 1.f / (1.f + expf(-a.beta[i]));
}
template <class Args>
__device__ __forceinline__ void load_gate(const Args& a, size_t i, int h, float& g, float& beta) {
  if (a.A_log == nullptr) {
    g = a.g[i];
    beta = a.beta[i];
  } else {
    gate_from_raw(a, i, h, g, beta);
  }
}
// The same with the mode fixed at compile time (kernels instantiated per mode).
template <bool kRaw, class Args>
__device__ __forceinline__ void load_gate_t(const Args& a, size_t i, int h, float& g, float& beta) {
  if constexpr (kRaw) {
    gate_from_raw(a, i, h, g, beta);
  } else {
    g = a.g[i];
    beta = a.beta[i];
  }
}

// State row of sequence n: n, or slots[n] with a slot map.  An id outside
// [0, num_slots) marks a padding sequence and gives -1 (no state is read or
// written for it).
template <class Args>
__device__ __forceinline__ int64_t state_row(const Args& a, int n) {
  if (a.slots == nullptr) return n;
  const int32_t s = a.slots[n];
  return (s >= 0 && s < a.num_slots) ? (int64_t)s : -1;
}

// SiLU, x * sigmoid(x) = x / (1 + exp(-x)): the gate of the RMSNorm epilogue
// (RMSNormGated of the "手撕Qwen3-Next" walkthrough, sections 一(一)1 and 6)
// and the activation after the causal conv (section 一(一)3).  Evaluated with
// the fast intrinsics (a few ulp; the accurate expf and IEEE division made the
// HBM-bound epilogue instruction-bound); the exponent is clamped at 80 so the
// divisor stays below the 2^126 limit of __fdividef (silu(-80) is -1.4e-33).
__device__ __forceinline__ float silu(float x) { return __fdividef(x, 1.f + __expf(fminf(-x, 80.f))); }

// Sequence bounds [start, end) of sequence n, clamped to 0 <= start <= end <=
// total_tokens.  cu_seqlens must be non-decreasing with cu[0] = 0 and
// cu[num_seqs] = total_tokens ([PTO] README, 参数说明: act_seq_len holds the
// cumulative lengths).  A violation that this sequence sees (its own bounds out
// of order or out of range, or a wrong first / last entry) is reported through
// the status word, and the clamped bounds keep every access inside the tensors.
template <class Args>
__device__ __forceinline__ void seq_bounds(const Args& a, int n, int64_t& start, int64_t& end) {
  if (a.cu) {
    const int64_t s = a.cu[n], e = a.cu[n + 1], T = a.total_tokens;
    const bool bad = s < 0 || e < s || e > T || (n == 0 && s != 0) || (n == a.num_seqs - 1 && e != T);
    start = s < 0 ? 0 : (s > T ? T : s);
    end = e < start ? start : (e > T ? T : e);
    if (bad) report_status(a.status, kStatusSeqlens);
  } else {
    start = (int64_t)n * a.uniform_len;
    end = start + a.uniform_len;
  }
}

}  // namespace gdn
