// Greedy acceptance of MTP draft tokens after the verify step.
//
// The verify step scores K + 1 new positions per sequence (GB10 page,
// ainews.surl.tw: MTP with K = 4 drafts at concurrency 1-128); row i of its
// logits predicts the token after new position i.  For every sequence:
//     target[i]   = first argmax of logits[b, i, :]            (i = 0 .. K)
//     n_accepted  = number of leading drafts with draft[i] == target[i]
//     next_token  = target[n_accepted]
// the draft -> verify -> accept loop of the speculative-decoding page
// (blog.hotdry.top, "Implementing kernel fusion in ATLAS speculative
// decoding").  One 256-thread CTA per logits row streams the row once with
// 16-byte loads (HBM-bound: the logits are read once, nothing else is large);
// the CTA that finishes a sequence's rows last (one atomic counter per
// sequence, no waiting) takes the acceptance decision and resets the counter.
#include <stdint.h>

#include "atlas_internal.cuh"

namespace atlas {
namespace {

// 256 threads: eight CTAs per SM, so the 640 rows of a 128-sequence, K = 4
// verify step are all resident at once (512-thread CTAs left a second, mostly
// empty wave: 47.1 vs 41.0 us)
constexpr int kThreads = 256;

// (value, index) with the larger value; on equal values the smaller index
__device__ __forceinline__ void better(float& v, int& i, float v2, int i2) {
  if (v2 > v || (v2 == v && i2 < i)) {
    v = v2;
    i = i2;
  }
}

template <typename T>
__device__ __forceinline__ float to_f32(T x);
template <>
__device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) {
  return __bfloat162float(x);
}

template <typename T>
__global__ void __launch_bounds__(kThreads) mtp_accept_kernel(const T* __restrict__ logits,
                                                              int vocab, int num_drafts,
                                                              const int32_t* __restrict__ drafts,
                                                              int32_t* targets,
                                                              int32_t* n_accepted,
                                                              int32_t* next_token,
                                                              int32_t* counters) {
  const int row = blockIdx.x;
  const int K1 = num_drafts + 1;
  const int b = row / K1;
  const T* x = logits + (size_t)row * vocab;
  const int tid = threadIdx.x;

  // each thread scans increasing indices, so a strictly greater value keeps
  // the first maximum of its share
  float best = -INFINITY;
  int idx = 0x7FFFFFFF;
  constexpr int V = 16 / sizeof(T);  // elements per 16-byte load
  const bool vec = (reinterpret_cast<uintptr_t>(x) % 16) == 0;
  int head = 0;
  if (vec) {
    const int nvec = vocab / V;
    const uint4* xv = reinterpret_cast<const uint4*>(x);
    for (int c = tid; c < nvec; c += kThreads) {
      const uint4 w = __ldcs(xv + c);  // streamed once: evict-first
      const T* e = reinterpret_cast<const T*>(&w);
#pragma unroll
      for (int k = 0; k < V; ++k) {
        const float v = to_f32<T>(e[k]);
        if (v > best) {
          best = v;
          idx = c * V + k;
        }
      }
    }
    head = nvec * V;
  }
  for (int j = head + tid; j < vocab; j += kThreads) {  // unaligned row or tail
    const float v = to_f32<T>(x[j]);
    if (v > best || (v == best && j < idx)) {
      best = v;
      idx = j;
    }
  }
  // block reduction of (value, index)
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float v2 = __shfl_xor_sync(0xFFFFFFFFu, best, o);
    const int i2 = __shfl_xor_sync(0xFFFFFFFFu, idx, o);
    better(best, idx, v2, i2);
  }
  __shared__ float s_v[kThreads / 32];
  __shared__ int s_i[kThreads / 32];
  __shared__ int s_last;
  if ((tid & 31) == 0) {
    s_v[tid >> 5] = best;
    s_i[tid >> 5] = idx;
  }
  __syncthreads();
  if (tid == 0) {
    for (int w = 1; w < kThreads / 32; ++w) better(best, idx, s_v[w], s_i[w]);
    if (idx == 0x7FFFFFFF) idx = 0;  // no value above -inf: the first index
    targets[row] = idx;
    __threadfence();
    s_last = (atomicAdd(counters + b, 1) == K1 - 1);
  }
  __syncthreads();
  if (tid != 0 || !s_last) return;
  // the last row of sequence b: take the acceptance decision
  __threadfence();
  const int32_t* tg = targets + (size_t)b * K1;
  int n = 0;
  while (n < num_drafts && __ldcg(drafts + (size_t)b * num_drafts + n) == __ldcg(tg + n)) ++n;
  n_accepted[b] = n;
  next_token[b] = __ldcg(tg + n);
  counters[b] = 0;  // ready for the next call on this stream
}

}  // namespace

cudaError_t launch_mtp_accept(const void* logits, int dtype, int batch, int num_drafts, int vocab,
                              const int32_t* drafts, int32_t* targets, int32_t* n_accepted,
                              int32_t* next_token, int32_t* counters, cudaStream_t stream) {
  const long long rows = (long long)batch * (num_drafts + 1);
  if (rows < 1 || rows > 0x7FFFFFFFLL) return cudaErrorInvalidValue;
  if (dtype == ATLAS_DTYPE_F32)
    mtp_accept_kernel<float><<<(unsigned)rows, kThreads, 0, stream>>>(
        static_cast<const float*>(logits), vocab, num_drafts, drafts, targets, n_accepted,
        next_token, counters);
  else
    mtp_accept_kernel<__nv_bfloat16><<<(unsigned)rows, kThreads, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(logits), vocab, num_drafts, drafts, targets,
        n_accepted, next_token, counters);
  return cudaGetLastError();
}

}  // namespace atlas
