// Fused rotary embedding + FP8 quantise + paged append, from the bf16 QKV
// projection output of the new tokens.
//
// The deep-dive page (Atlas: Rust/CUDA LLM inference engine, ainews.cool,
// "Kernel fusion" paragraph) fuses the steps of a transformer block into one
// kernel; this is the step in front of paged decode.  For every new token t of
// sequence b (position pos = start_pos[b] + t) and every head of its
// projection row [Hq query | Hkv key | Hkv value heads] x D (bf16):
//   * query and key heads are rotated ("rotate half": element i < D/2 pairs
//     with i + D/2; with c = cos_sin[pos][i], s = cos_sin[pos][D/2 + i]
//         out[i] = x[i] c - x[i + D/2] s,   out[i + D/2] = x[i + D/2] c + x[i] s
//     in float32, every product and sum rounded separately -- no fused
//     multiply-add -- so the value that decides an FP8 code is one exact
//     float32 number);
//   * the rotated query is written as bf16 (round to nearest even);
//   * the rotated key and the value are quantised to E4M3 with the per-KV-head
//     scale (IEEE division, round to nearest even, saturating) and scattered
//     into their pages exactly as atlas_fp8_kv_append does.
// HBM-bound: each projection row is read once (2 bytes per element), the
// cos/sin row of a position is read once per window of 16 tokens into shared
// memory and shared by all heads, and each element leaves as 2 (query) or 1
// (key, value) bytes.
#include "atlas_internal.cuh"

namespace atlas {
namespace {

constexpr int kThreads = 256;
constexpr int kWin = 16;   // tokens per CTA: one 16-slot V group when aligned

// CTA = a window of 16 consecutive new tokens of one sequence, all heads: the
// cos/sin rows of the window are read once into shared memory; query and key
// heads are rotated in (token, head, 8 column pairs) tasks, four per thread
// and pass with their loads issued first; the value heads are quantised two
// head dimensions per task -- 16 tokens of a dimension form one 16-byte group
// row of a V page.
template <int D>
__global__ void __launch_bounds__(kThreads) rope_append_kernel(const RopeAppendParams p) {
  constexpr int TPR = D / 16;          // tasks per head row: 8 column pairs each
  constexpr int H2 = D / 2;
  __shared__ __align__(16) float s_cs[kWin][D];
  __shared__ int s_ok[kWin];           // position inside the table
  __shared__ int s_page[kWin];         // page of the token (-1: K/V not stored)
  const int heads = p.Hq + 2 * p.Hkv;
  const int n_win = (p.n_new + kWin - 1) / kWin;
  const int b = blockIdx.x / n_win, w0 = (blockIdx.x % n_win) * kWin;
  const int n_tok = min(kWin, p.n_new - w0);
  const int start = __ldg(p.start_pos + b);
  const int tid = threadIdx.x;

  if (tid < kWin) {
    const int pos = start + w0 + tid;
    int ok = 0, page = -1;
    if (tid < n_tok) {
      ok = pos >= 0 && pos < p.max_pos;
      if (ok) {
        const int blk = pos / p.ps;
        if (blk < p.max_blocks) page = __ldg(p.block_table + (size_t)b * p.max_blocks + blk);
        if (page < 0 || page >= p.num_pages) page = -1;
      }
      if (!ok || page < 0) atomicOr(p.err, ATLAS_DEVERR_APPEND);
    }
    s_ok[tid] = ok;
    s_page[tid] = ok ? page : -1;
  }
  __syncthreads();
  for (int idx = tid; idx < kWin * (D / 4); idx += kThreads) {  // the window's cos/sin rows
    const int t = idx / (D / 4), c4 = idx % (D / 4);
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (t < n_tok && s_ok[t])
      v = __ldg(reinterpret_cast<const float4*>(p.cos_sin + (size_t)(start + w0 + t) * D) + c4);
    *reinterpret_cast<float4*>(&s_cs[t][4 * c4]) = v;
  }
  __syncthreads();

  // ---- query and key heads: rotate; queries -> bf16, keys -> E4M3 pages.
  // Four tasks per thread and pass: their loads go out before any of their
  // arithmetic, so each thread keeps eight 16-byte loads in flight
  const int qk_heads = p.Hq + p.Hkv;
  const int n_qk = n_tok * qk_heads * TPR;
  constexpr int U = 4;
  for (int base = 0; base < n_qk; base += U * kThreads) {
    uint4 la[U], lz[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int task = base + u * kThreads + tid;
      la[u] = make_uint4(0u, 0u, 0u, 0u);
      lz[u] = la[u];
      if (task < n_qk) {
        const int c = task % TPR, th = task / TPR;
        const int head = th % qk_heads, t = th / qk_heads;
        if (s_ok[t]) {
          const size_t tok = (size_t)b * p.n_new + w0 + t;
          const __nv_bfloat16* src = p.qkv + (tok * heads + head) * D;
          la[u] = __ldg(reinterpret_cast<const uint4*>(src + 8 * c));
          lz[u] = __ldg(reinterpret_cast<const uint4*>(src + H2 + 8 * c));
        }
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int task = base + u * kThreads + tid;
      if (task >= n_qk) break;
      const int c = task % TPR;                 // columns [8c, 8c+8) and [D/2+8c, D/2+8c+8)
      const int th = task / TPR;
      const int head = th % qk_heads, t = th / qk_heads;
      if (!s_ok[t]) continue;
      const size_t tok = (size_t)b * p.n_new + w0 + t;
      float x[16];
      {
        const uint32_t wa[4] = {la[u].x, la[u].y, la[u].z, la[u].w};
        const uint32_t wz[4] = {lz[u].x, lz[u].y, lz[u].z, lz[u].w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          x[2 * k] = __uint_as_float(wa[k] << 16);
          x[2 * k + 1] = __uint_as_float(wa[k] & 0xFFFF0000u);
          x[8 + 2 * k] = __uint_as_float(wz[k] << 16);
          x[8 + 2 * k + 1] = __uint_as_float(wz[k] & 0xFFFF0000u);
        }
      }
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const float co = s_cs[t][8 * c + k], si = s_cs[t][H2 + 8 * c + k];
        const float x1 = x[k], x2 = x[8 + k];
        x[k] = __fsub_rn(__fmul_rn(x1, co), __fmul_rn(x2, si));
        x[8 + k] = __fadd_rn(__fmul_rn(x2, co), __fmul_rn(x1, si));
      }
      if (head < p.Hq) {  // rotated query -> bf16
        __nv_bfloat16* dst = p.q_out + (tok * p.Hq + head) * D;
        uint32_t w[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const __nv_bfloat162 v2 = __floats2bfloat162_rn(x[2 * k], x[2 * k + 1]);
          w[k] = *reinterpret_cast<const uint32_t*>(&v2);
        }
        *reinterpret_cast<uint4*>(dst + 8 * c) = make_uint4(w[0], w[1], w[2], w[3]);
        *reinterpret_cast<uint4*>(dst + H2 + 8 * c) = make_uint4(w[4], w[5], w[6], w[7]);
        continue;
      }
      const int page = s_page[t];
      if (page < 0) continue;
      const int h = head - p.Hq;
      const uint4 codes = quantize16_e4m3(x, __ldg(p.k_scale + h));
      const int slot = (start + w0 + t) % p.ps;
      // dims [8c, 8c + 8) and [D/2 + 8c, ...): half of 16-byte chunk 8c / 16 and
      // of chunk (D/2 + 8c) / 16, placed by the K page layout
      uint8_t* rowp = p.k_pages + (((size_t)page * p.Hkv + h) * p.ps + slot) * D;
      const int j0 = (8 * c) / 16, j1 = (H2 + 8 * c) / 16, sub = (8 * c) % 16;
      *reinterpret_cast<uint2*>(rowp + 16 * k_chunk_pos(D, slot, j0) + sub) =
          make_uint2(codes.x, codes.y);
      *reinterpret_cast<uint2*>(rowp + 16 * k_chunk_pos(D, slot, j1) + sub) =
          make_uint2(codes.z, codes.w);
    }
  }

  // ---- value heads: head dimensions of the window's 16 tokens
  const int p0 = start + w0;
  // an aligned window is one 16-slot group of one page: whole-row stores when
  // every token of it is stored (positions increase, so the last one decides
  // the table bound)
  const bool whole_group = n_tok == kWin && (p0 % 16) == 0 && s_page[0] >= 0 && s_ok[kWin - 1];
  // Two adjacent head dimensions per task (one 4-byte load per token covers
  // both), their 16 tokens' loads issued before any division
  for (int task = tid; task < p.Hkv * (D / 2); task += kThreads) {
    const int h = task / (D / 2), d = 2 * (task % (D / 2));
    const float vs = __ldg(p.v_scale + h);
    uint32_t raw[kWin];
#pragma unroll
    for (int t = 0; t < kWin; ++t) {
      raw[t] = 0u;
      if (t < n_tok) {
        const size_t tok = (size_t)b * p.n_new + w0 + t;
        raw[t] = __ldg(reinterpret_cast<const uint32_t*>(
            p.qkv + (tok * heads + p.Hq + p.Hkv + h) * D + d));
      }
    }
#pragma unroll
    for (int e = 0; e < 2; ++e) {  // dimension d + e
      uint32_t code[kWin];
#pragma unroll
      for (int t = 0; t < kWin; t += 2) {
        const float x0 = __uint_as_float(e ? (raw[t] & 0xFFFF0000u) : (raw[t] << 16));
        const float x1 = __uint_as_float(e ? (raw[t + 1] & 0xFFFF0000u) : (raw[t + 1] << 16));
        const float y0 = t < n_tok ? __fdiv_rn(x0, vs) : 0.f;
        const float y1 = t + 1 < n_tok ? __fdiv_rn(x1, vs) : 0.f;
        const uint32_t pr = __nv_cvt_float2_to_fp8x2(make_float2(y0, y1), __NV_SATFINITE,
                                                     __NV_E4M3);
        code[t] = pr & 0xFFu;
        code[t + 1] = (pr >> 8) & 0xFFu;
      }
      const size_t head_page0 = (size_t)max(s_page[0], 0) * p.Hkv + h;
      if (whole_group) {  // word c of a group row holds slots 2c, 2c+1, 2c+8, 2c+9
        uint32_t w[4];
#pragma unroll
        for (int cc = 0; cc < 4; ++cc)
          w[cc] = code[2 * cc] | (code[2 * cc + 1] << 8) | (code[2 * cc + 8] << 16) |
                  (code[2 * cc + 9] << 24);
        uint8_t* dst =
            p.v_pages + (head_page0 * (p.ps / 16) + (p0 % p.ps) / 16) * (16 * D) + 16 * (d + e);
        *reinterpret_cast<uint4*>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
      } else {
#pragma unroll
        for (int t = 0; t < kWin; ++t) {
          const int pg = s_page[t];
          if (t >= n_tok || pg < 0) continue;
          const int slot = (p0 + t) % p.ps;
          const int g = slot % 16;
          const int byte = 4 * ((g & 7) >> 1) + 2 * (g >> 3) + (g & 1);
          p.v_pages[(((size_t)pg * p.Hkv + h) * (p.ps / 16) + slot / 16) * (16 * D) +
                    16 * (d + e) + byte] = (uint8_t)code[t];
        }
      }
    }
  }
}

}  // namespace

cudaError_t launch_rope_append(const RopeAppendParams& p, cudaStream_t stream) {
  if (p.batch == 0 || p.n_new == 0) return cudaSuccess;
  const long long grid = (long long)p.batch * ((p.n_new + kWin - 1) / kWin);
  if (grid > 0x7FFFFFFFLL) return cudaErrorInvalidValue;
  if (p.D == 128)
    rope_append_kernel<128><<<(unsigned)grid, kThreads, 0, stream>>>(p);
  else if (p.D == 64)
    rope_append_kernel<64><<<(unsigned)grid, kThreads, 0, stream>>>(p);
  else
    return cudaErrorInvalidValue;
  return cudaGetLastError();
}

}  // namespace atlas
