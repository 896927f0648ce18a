// FP8 page append: quantise new K/V rows to E4M3 with a per-KV-head scale and
// scatter them into their pages through the block table.
//
// Source: the FP8 KV quantisation with scale factors of the Atlas deep-dive
// (ainews.cool, "Quantisation" paragraph) and the paged FP8 KV cache of the
// GB10 page (ainews.surl.tw).  Encoding reading: y = fp32(x) / fp32(scale[h])
// as an IEEE round-to-nearest division (__fdiv_rn, never a reciprocal
// multiply), then round-to-nearest-even to E4M3 with saturation to +-448
// (cvt.rn.satfinite), sign of zero kept.  The result must be bit-exact with
// that definition.
//
// Finer-grained mode (k_tok_scale != nullptr): each token's row of each KV
// head gets its own dynamic scale amax / 448, stored at [page][head][slot] of
// the scale arrays, and the head's bound of the V scales is raised to it.
//
// Page layouts: K pages are token-major [P][Hkv][ps][D] (with D = 128 the
// 16-byte chunk j of slot s sits at chunk position j XOR (s % 8)); V pages are kept in
// groups of 16 slots, head-dim-major inside a group: [P][Hkv][ps/16][D][16]
// (16 consecutive tokens of one head dimension adjacent), slot t of a group at
// byte 4*((t%8)/2) + 2*(t/8) + t%2 (bytes 4c..4c+3 hold slots 2c, 2c+1, 2c+8,
// 2c+9, the token order of the decode kernel's P fragments).
// Memory-bound: per element 4 (f32) or 2 (bf16) bytes read, 1 byte written.
// A CTA owns 16 consecutive new tokens of one (sequence, KV head), D threads.
// K: thread (token, chunk) quantises 16 consecutive elements of one token row
// and stores them as one 16-byte write.  V: thread d takes head dimension d of
// the 16 tokens (every load instruction reads one token row across the CTA,
// coalesced), so the group row of dimension d -- 16 codes in the group's slot
// order -- is formed in registers and leaves as one 16-byte write when the 16
// tokens fill one 16-slot group of a page exactly (the cache-fill case); the
// few tokens of a decode step are stored as single bytes.
#include "atlas_internal.cuh"

namespace atlas {
namespace {

constexpr int kTok = 16;  // tokens per CTA (one 16-slot V group when aligned)

// Dynamic per-(token, KV head) scale of the finer-grained mode: the largest
// |x| over the token's D elements (held 16 per thread by the CH = D / 16
// consecutive threads of the token), divided by 448 (IEEE division); 1 for an
// all-zero row.  Every thread of the warp takes part in the shuffles.
template <int CH>
__device__ __forceinline__ float token_row_scale(const float (&x)[16]) {
  float a = 0.f;
#pragma unroll
  for (int k = 0; k < 16; ++k) a = fmaxf(a, fabsf(x[k]));
#pragma unroll
  for (int o = 1; o < CH; o <<= 1) a = fmaxf(a, __shfl_xor_sync(0xFFFFFFFFu, a, o));
  return a > 0.f ? __fdiv_rn(a, 448.f) : 1.f;
}

template <int D, bool TS>
__global__ void __launch_bounds__(D) fp8_append_kernel(const AppendParams p) {
  constexpr int CH = D / 16;  // 16-element chunks per row
  constexpr int NW = D / 32;  // warps
  __shared__ int s_page[kTok];
  __shared__ float s_amax[NW][kTok];
  const int n_tiles = (p.n_new + kTok - 1) / kTok;
  const int tile = blockIdx.x % n_tiles;
  const int bh = blockIdx.x / n_tiles;
  const int h = bh % p.Hkv, b = bh / p.Hkv;
  const int t0 = tile * kTok;
  const int n_tok = min(kTok, p.n_new - t0);
  const int start = __ldg(p.start_pos + b);
  const int tid = threadIdx.x;
  const int lt = tid / CH, j = tid % CH;  // K: token within the tile, chunk

  if (tid < kTok) {  // page of each token of the tile (-1: not written, flagged)
    int page = -1;
    const int pos = start + t0 + tid;
    if (tid < n_tok) {
      const int blk = pos / p.ps;
      if (pos >= 0 && blk < p.max_blocks) {
        page = __ldg(p.block_table + (size_t)b * p.max_blocks + blk);
        if (page < 0 || page >= p.num_pages) page = -1;
      }
      if (page < 0) atomicOr(p.err, ATLAS_DEVERR_APPEND);
    }
    s_page[tid] = page;
  }

  // ---- V, one head dimension per thread: element d of the tile's 16 tokens
  // (each load instruction reads one token's row across the CTA: coalesced),
  // quantised and packed in the 16-slot group order -- one 16-byte store per
  // thread when the tile is exactly one group of one page
  const int d = tid;
  float xv[kTok];
#pragma unroll
  for (int t = 0; t < kTok; ++t) {
    xv[t] = 0.f;
    if (t < n_tok) {
      const size_t e = (((size_t)b * p.n_new + t0 + t) * p.Hkv + h) * D + d;
      xv[t] = (p.dtype == ATLAS_DTYPE_F32)
                  ? __ldg(static_cast<const float*>(p.v_new) + e)
                  : __bfloat162float(__ldg(static_cast<const __nv_bfloat16*>(p.v_new) + e));
    }
  }
  float vsc[kTok];
  if constexpr (TS) {  // per-token scales: the row maximum over all D threads
#pragma unroll
    for (int t = 0; t < kTok; ++t) {
      float a = fabsf(xv[t]);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xFFFFFFFFu, a, o));
      if ((tid & 31) == 0) s_amax[tid >> 5][t] = a;
    }
  }
  __syncthreads();  // s_page (and s_amax) ready
  if constexpr (TS) {
#pragma unroll
    for (int t = 0; t < kTok; ++t) {
      float a = s_amax[0][t];
#pragma unroll
      for (int w = 1; w < NW; ++w) a = fmaxf(a, s_amax[w][t]);
      vsc[t] = a > 0.f ? __fdiv_rn(a, 448.f) : 1.f;
    }
  } else {
    const float s0 = __ldg(p.v_scale + h);
#pragma unroll
    for (int t = 0; t < kTok; ++t) vsc[t] = s0;
  }
  uint32_t code[kTok];
#pragma unroll
  for (int t = 0; t < kTok; t += 2) {
    const float y0 = __fdiv_rn(xv[t], vsc[t]), y1 = __fdiv_rn(xv[t + 1], vsc[t + 1]);
    const uint32_t pr = __nv_cvt_float2_to_fp8x2(make_float2(y0, y1), __NV_SATFINITE, __NV_E4M3);
    code[t] = pr & 0xFFu;
    code[t + 1] = (pr >> 8) & 0xFFu;
  }
  const int p0 = start + t0;
  const bool whole_group = n_tok == kTok && (p0 % 16) == 0 && s_page[0] >= 0;
  if (whole_group) {
    // slot t of the group sits at byte 4*((t%8)/2) + 2*(t/8) + t%2: word c
    // holds slots 2c, 2c+1, 2c+8, 2c+9
    uint32_t w[4];
#pragma unroll
    for (int c = 0; c < 4; ++c)
      w[c] = code[2 * c] | (code[2 * c + 1] << 8) | (code[2 * c + 8] << 16) |
             (code[2 * c + 9] << 24);
    const size_t head_page = (size_t)s_page[0] * p.Hkv + h;
    uint8_t* dst = p.v_pages + (head_page * (p.ps / 16) + (p0 % p.ps) / 16) * (16 * D) + 16 * d;
    *reinterpret_cast<uint4*>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
  } else {  // byte stores for the valid tokens (a decode step's few tokens)
#pragma unroll
    for (int t = 0; t < kTok; ++t) {
      const int pg = s_page[t];
      if (t >= n_tok || pg < 0) continue;
      const int slot = (p0 + t) % p.ps;
      const int g = slot % 16;
      const int byte = 4 * ((g & 7) >> 1) + 2 * (g >> 3) + (g & 1);
      const size_t head_page = (size_t)pg * p.Hkv + h;
      p.v_pages[(head_page * (p.ps / 16) + slot / 16) * (16 * D) + 16 * d + byte] =
          (uint8_t)code[t];
    }
  }
  if (TS && d < n_tok && s_page[d] >= 0) {  // thread t < 16 stores token t's V scale
    float a = s_amax[0][d];
#pragma unroll
    for (int w = 1; w < NW; ++w) a = fmaxf(a, s_amax[w][d]);
    const float sc = a > 0.f ? __fdiv_rn(a, 448.f) : 1.f;
    const int slot = (p0 + d) % p.ps;
    p.v_tok_scale[((size_t)s_page[d] * p.Hkv + h) * p.ps + slot] = sc;
    // positive floats order like their bit patterns: the head's running bound
    // of the per-token V scales
    atomicMax(reinterpret_cast<int*>(p.v_scale_bound + h), __float_as_int(sc));
  }

  // ---- K, 16 consecutive elements of one token row per thread (one
  // 16-byte store of codes each)
  const int pos = start + t0 + lt;
  const int page = s_page[lt];
  const bool ok = lt < n_tok && page >= 0;
  float x[16];
  if (ok) {
    load16_as_f32(p.k_new, (((size_t)b * p.n_new + t0 + lt) * p.Hkv + h) * D + 16 * j, p.dtype,
                  x);
  } else {
#pragma unroll
    for (int k = 0; k < 16; ++k) x[k] = 0.f;
  }
  const float ks = TS ? token_row_scale<CH>(x) : __ldg(p.k_scale + h);
  if (ok) {
    const size_t head_page = (size_t)page * p.Hkv + h;
    const int slot = pos % p.ps;
    store16_k(p.k_pages, head_page, D, p.ps, slot, j, quantize16_e4m3(x, ks));
    if (TS && j == 0) p.k_tok_scale[head_page * p.ps + slot] = ks;
  }
}

}  // namespace

cudaError_t launch_fp8_append(const AppendParams& p, int num_sms, cudaStream_t stream) {
  (void)num_sms;
  if (p.batch == 0 || p.n_new == 0) return cudaSuccess;
  const long long n_tiles = (p.n_new + kTok - 1) / kTok;
  const long long blocks = n_tiles * p.Hkv * p.batch;
  if (blocks > 0x7FFFFFFFLL) return cudaErrorInvalidValue;
  const bool ts = p.k_tok_scale != nullptr;
  if (p.D == 128) {
    if (ts)
      fp8_append_kernel<128, true><<<(unsigned)blocks, 128, 0, stream>>>(p);
    else
      fp8_append_kernel<128, false><<<(unsigned)blocks, 128, 0, stream>>>(p);
  } else if (p.D == 64) {
    if (ts)
      fp8_append_kernel<64, true><<<(unsigned)blocks, 64, 0, stream>>>(p);
    else
      fp8_append_kernel<64, false><<<(unsigned)blocks, 64, 0, stream>>>(p);
  } else {
    return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace atlas
