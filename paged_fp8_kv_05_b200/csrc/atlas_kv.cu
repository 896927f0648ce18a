// C-ABI layer of libatlas_kv.so: argument checks, launch planning and the
// entry points declared in include/atlas_kv.h.  Owns no device memory.
#include <math.h>
#include <stdlib.h>
#include <string.h>

#include <new>

#include "atlas_internal.cuh"

struct atlas_kv_pool {
  int32_t num_pages, page_size, num_kv_heads, head_dim;
  uint8_t* k_pages;
  uint8_t* v_pages;
  const float* k_scale;
  const float* v_scale;
  int32_t max_batch, max_q_len, num_q_heads;
  uint8_t* workspace;
  size_t workspace_bytes;
  int32_t split_override;
  int32_t stages_override;
  int32_t waves_override;
  int32_t partition_override;
  int32_t rows_override;
  int32_t kernel_override; // atlas::kKernel*
  int32_t wait_limit_us;   // 0: the default limit of every bounded wait
  int32_t test_skip_unit;  // -1: normal; >= 0: lost-copy injection (tests only)
  size_t counters_bytes;  // largest counter block any accepted call uses
};

namespace {

constexpr size_t kAlign = 256;
constexpr int kDefaultSms = 148;          // B200; used only when no device is visible
constexpr int kMinSplit = 64;             // 4 warps x 16-token units
constexpr int kMaxSplit = 8192;

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int device_sm_count() {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    cudaGetLastError();
    return kDefaultSms;
  }
  if (cached[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
      cudaGetLastError();
      return kDefaultSms;
    }
    cached[dev] = n;
  }
  return cached[dev];
}

// Workspace of one call: [error word][counters][log2-sum-exp][O partials].
struct WsLayout {
  size_t counters, lse, o, total;
};
WsLayout ws_layout(const atlas::DecodeLaunch& L, int head_dim) {
  WsLayout w;
  w.counters = kAlign;
  const size_t cnt = align_up((size_t)L.segs * sizeof(int32_t), kAlign);
  w.lse = w.counters + cnt;
  const size_t rows = (size_t)L.slots * L.rows_per_cta;
  w.o = w.lse + align_up(rows * sizeof(float), kAlign);
  w.total = w.o + align_up(rows * head_dim * sizeof(float), kAlign);
  return w;
}

// Split-KV partition (A1): splits of each segment handed to SMs by the
// hardware, or balanced ranges of 32-token units (see atlas::plan_decode).
// The split / range length adapts to the lengths and the SM count -- the
// "block size adapted to sequence length and architecture" of the Atlas
// deep-dive's attention paragraph.
atlas::DecodeLaunch make_plan(const atlas_kv_pool* pool, int batch, int num_q_heads, int q_len,
                              int max_seq_len, int sms, bool fit, bool* tc, bool varlen = false) {
  *tc = atlas::use_tc_kernel(pool->kernel_override, pool->head_dim, q_len,
                             num_q_heads / pool->num_kv_heads);
  if (*tc)
    return atlas::plan_decode_tc(batch, num_q_heads, pool->num_kv_heads, q_len, max_seq_len, sms,
                                 pool->split_override, pool->stages_override,
                                 pool->waves_override > 0 ? pool->waves_override : 1);
  // ragged q_len: the grid partition (a CTA serves one segment, so row blocks
  // past a sequence's rows cost nothing)
  atlas::DecodeLaunch L = atlas::plan_decode(batch, num_q_heads, pool->num_kv_heads, q_len,
                                             max_seq_len, sms, pool->split_override,
                                             pool->stages_override,
                                             varlen ? atlas::kPartitionGrid
                                                    : pool->partition_override,
                                             pool->waves_override > 0 ? pool->waves_override : 1,
                                             pool->rows_override);
  if (fit && pool->split_override == 0 && !L.grid_mode) {
    const int R = q_len * (num_q_heads / pool->num_kv_heads);
    atlas::decode_fp8_fit_grid(pool->head_dim, R < L.rows_per_cta ? R : L.rows_per_cta, sms, L);
  }
  return L;
}

bool device_present() {
  int cnt = 0;
  if (cudaGetDeviceCount(&cnt) != cudaSuccess || cnt <= 0) {
    cudaGetLastError();
    return false;
  }
  return true;
}

}  // namespace

extern "C" {

const char* atlas_version(void) { return "0.1.0"; }

const char* atlas_status_string(atlas_status_t s) {
  switch (s) {
    case ATLAS_OK: return "ok";
    case ATLAS_ERR_INVALID_ARG: return "invalid argument";
    case ATLAS_ERR_UNSUPPORTED: return "unsupported shape";
    case ATLAS_ERR_WORKSPACE: return "workspace too small";
    case ATLAS_ERR_CUDA: return "CUDA runtime error";
    case ATLAS_ERR_DEVICE_CHECK: return "device-side check failed";
  }
  return "unknown status";
}

size_t atlas_kv_workspace_bytes(int32_t max_batch, int32_t max_q_len, int32_t num_q_heads,
                                int32_t num_kv_heads, int32_t head_dim, int32_t max_seq_len,
                                int32_t min_split_tokens) {
  if (max_batch < 0 || max_q_len < 1 || num_q_heads < 1 || num_kv_heads < 1 || max_seq_len < 0)
    return 0;
  if (num_q_heads % num_kv_heads != 0) return 0;
  if (head_dim != 64 && head_dim != 128) return 0;
  if (min_split_tokens < 0) return 0;
  const int sms = device_present() ? device_sm_count() : kDefaultSms;
  size_t need = 0;
  for (int ql = 1; ql <= max_q_len; ++ql) {
    const int msl = max_seq_len > ql ? max_seq_len : ql;
    // both partitions, automatic and with the finest split override the caller
    // will set
    for (int part : {atlas::kPartitionGrid, atlas::kPartitionBalanced})
      for (int split : {0, min_split_tokens}) {
        const atlas::DecodeLaunch L =
            atlas::plan_decode(max_batch, num_q_heads, num_kv_heads, ql, msl, sms, split, 0, part);
        const size_t t = ws_layout(L, head_dim).total;
        if (t > need) need = t;
      }
    // the tensor-core kernel's plans (head_dim 128)
    if (head_dim == 128)
      for (int split : {0, min_split_tokens}) {
        const atlas::DecodeLaunch L =
            atlas::plan_decode_tc(max_batch, num_q_heads, num_kv_heads, ql, msl, sms, split, 0);
        const size_t t = ws_layout(L, head_dim).total;
        if (t > need) need = t;
      }
    // the counter block of the finest row grouping (4 rows per block)
    const atlas::DecodeLaunch L4 = atlas::plan_decode(max_batch, num_q_heads, num_kv_heads, ql,
                                                      msl, sms, 0, 0, atlas::kPartitionGrid, 1, 4);
    const size_t c4 = kAlign + align_up((size_t)L4.segs * sizeof(int32_t), kAlign);
    if (c4 > need) need = c4;
  }
  return need;
}

atlas_status_t atlas_kv_pool_create(atlas_kv_pool_t** out, int32_t num_pages, int32_t page_size,
                                    int32_t num_kv_heads, int32_t head_dim, void* k_pages,
                                    void* v_pages, const float* k_scale, const float* v_scale,
                                    int32_t max_batch, int32_t max_q_len, int32_t num_q_heads,
                                    void* workspace, size_t workspace_bytes) {
  if (!out) return ATLAS_ERR_INVALID_ARG;
  *out = nullptr;
  if (num_pages < 1 || num_kv_heads < 1 || max_batch < 0 || max_q_len < 1 || num_q_heads < 1)
    return ATLAS_ERR_INVALID_ARG;
  if (page_size < 16 || page_size > 1024 || page_size % 16 != 0) return ATLAS_ERR_UNSUPPORTED;
  if (head_dim != 64 && head_dim != 128) return ATLAS_ERR_UNSUPPORTED;
  if (num_q_heads % num_kv_heads != 0) return ATLAS_ERR_INVALID_ARG;
  if (!k_pages || !v_pages || !k_scale || !v_scale || !workspace) return ATLAS_ERR_INVALID_ARG;
  if (!aligned(k_pages, 16) || !aligned(v_pages, 16) || !aligned(workspace, kAlign))
    return ATLAS_ERR_INVALID_ARG;
  size_t counters_bytes = 0;
  for (int ql = 1; ql <= max_q_len; ++ql) {
    // the most segments any row grouping makes: 4 rows per block
    const atlas::DecodeLaunch L = atlas::plan_decode(max_batch, num_q_heads, num_kv_heads, ql, ql,
                                                     kDefaultSms, 0, 0, atlas::kPartitionAuto, 1,
                                                     4);
    const size_t c = align_up((size_t)L.segs * sizeof(int32_t), kAlign);
    if (c > counters_bytes) counters_bytes = c;
  }
  if (workspace_bytes < kAlign + counters_bytes) return ATLAS_ERR_WORKSPACE;
  atlas_kv_pool* p = new (std::nothrow) atlas_kv_pool;
  if (!p) return ATLAS_ERR_INVALID_ARG;
  p->num_pages = num_pages;
  p->page_size = page_size;
  p->num_kv_heads = num_kv_heads;
  p->head_dim = head_dim;
  p->k_pages = static_cast<uint8_t*>(k_pages);
  p->v_pages = static_cast<uint8_t*>(v_pages);
  p->k_scale = k_scale;
  p->v_scale = v_scale;
  p->max_batch = max_batch;
  p->max_q_len = max_q_len;
  p->num_q_heads = num_q_heads;
  p->workspace = static_cast<uint8_t*>(workspace);
  p->workspace_bytes = workspace_bytes;
  p->split_override = 0;
  p->stages_override = 0;
  p->waves_override = 0;
  p->partition_override = 0;
  p->rows_override = 0;
  p->kernel_override = 0;
  p->wait_limit_us = 0;
  p->test_skip_unit = -1;
  p->counters_bytes = counters_bytes;
  *out = p;
  return ATLAS_OK;
}

atlas_status_t atlas_kv_pool_destroy(atlas_kv_pool_t* pool) {
  delete pool;
  return ATLAS_OK;
}

atlas_status_t atlas_kv_pool_set_split_tokens(atlas_kv_pool_t* pool, int32_t split_tokens) {
  if (!pool) return ATLAS_ERR_INVALID_ARG;
  if (split_tokens != 0 &&
      (split_tokens < kMinSplit || split_tokens > kMaxSplit || split_tokens % kMinSplit != 0))
    return ATLAS_ERR_INVALID_ARG;
  pool->split_override = split_tokens;
  return ATLAS_OK;
}

atlas_status_t atlas_kv_pool_set_option(atlas_kv_pool_t* pool, int32_t option, int32_t value) {
  if (!pool) return ATLAS_ERR_INVALID_ARG;
  switch (option) {
    case ATLAS_OPT_SPLIT_TOKENS:
      return atlas_kv_pool_set_split_tokens(pool, value);
    case ATLAS_OPT_STAGES:
      if (value != 0 && value != 2 && value != 3) return ATLAS_ERR_INVALID_ARG;
      pool->stages_override = value;
      return ATLAS_OK;
    case ATLAS_OPT_WAVES:
      if (value < 0 || value > 8) return ATLAS_ERR_INVALID_ARG;
      pool->waves_override = value;
      return ATLAS_OK;
    case ATLAS_OPT_PARTITION:
      if (value < 0 || value > 2) return ATLAS_ERR_INVALID_ARG;
      pool->partition_override = value;
      return ATLAS_OK;
    case ATLAS_OPT_ROWS_PER_CTA:
      if (value != 0 && value != 4 && value != 8 && value != 16 && value != 32 && value != 64)
        return ATLAS_ERR_INVALID_ARG;
      pool->rows_override = value;
      return ATLAS_OK;
    case ATLAS_OPT_KERNEL:
      if (value < 0 || value > 2) return ATLAS_ERR_INVALID_ARG;
      if (value == atlas::kKernelTc && pool->head_dim != 128) return ATLAS_ERR_UNSUPPORTED;
      pool->kernel_override = value;
      return ATLAS_OK;
    case ATLAS_OPT_WAIT_LIMIT_US:
      if (value < 0 || value > 10 * 1000 * 1000) return ATLAS_ERR_INVALID_ARG;
      pool->wait_limit_us = value;
      return ATLAS_OK;
    case ATLAS_OPT_TEST_SKIP_UNIT:
      if (value < -1) return ATLAS_ERR_INVALID_ARG;
      pool->test_skip_unit = value;
      return ATLAS_OK;
  }
  return ATLAS_ERR_INVALID_ARG;
}

static atlas_status_t append_impl(const atlas_kv_pool_t* pool, const void* k_new,
                                  const void* v_new, int32_t dtype, const int32_t* block_table,
                                  int32_t max_blocks_per_seq, const int32_t* start_pos,
                                  int32_t batch, int32_t n_new, float* k_tok_scale,
                                  float* v_tok_scale, float* v_scale_bound, void* stream) {
  if (!pool) return ATLAS_ERR_INVALID_ARG;
  if (batch < 0 || n_new < 0 || max_blocks_per_seq < 1) return ATLAS_ERR_INVALID_ARG;
  if (dtype != ATLAS_DTYPE_F32 && dtype != ATLAS_DTYPE_BF16) return ATLAS_ERR_INVALID_ARG;
  if (batch == 0 || n_new == 0) return ATLAS_OK;
  if (!k_new || !v_new || !block_table || !start_pos) return ATLAS_ERR_INVALID_ARG;
  if (!aligned(k_new, 16) || !aligned(v_new, 16)) return ATLAS_ERR_INVALID_ARG;
  atlas::AppendParams p{};
  p.k_new = k_new;
  p.v_new = v_new;
  p.dtype = dtype;
  p.k_pages = pool->k_pages;
  p.v_pages = pool->v_pages;
  p.k_scale = pool->k_scale;
  p.v_scale = pool->v_scale;
  p.block_table = block_table;
  p.start_pos = start_pos;
  p.err = reinterpret_cast<int32_t*>(pool->workspace);
  p.batch = batch;
  p.n_new = n_new;
  p.Hkv = pool->num_kv_heads;
  p.D = pool->head_dim;
  p.ps = pool->page_size;
  p.num_pages = pool->num_pages;
  p.max_blocks = max_blocks_per_seq;
  p.k_tok_scale = k_tok_scale;
  p.v_tok_scale = v_tok_scale;
  p.v_scale_bound = v_scale_bound;
  cudaError_t e = atlas::launch_fp8_append(p, device_sm_count(), static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? ATLAS_OK : ATLAS_ERR_CUDA;
}

atlas_status_t atlas_fp8_kv_append(const atlas_kv_pool_t* pool, const void* k_new,
                                   const void* v_new, int32_t dtype, const int32_t* block_table,
                                   int32_t max_blocks_per_seq, const int32_t* start_pos,
                                   int32_t batch, int32_t n_new, void* stream) {
  return append_impl(pool, k_new, v_new, dtype, block_table, max_blocks_per_seq, start_pos,
                     batch, n_new, nullptr, nullptr, nullptr, stream);
}

atlas_status_t atlas_fp8_kv_append_tokscale(const atlas_kv_pool_t* pool, const void* k_new,
                                            const void* v_new, int32_t dtype,
                                            const int32_t* block_table, int32_t max_blocks_per_seq,
                                            const int32_t* start_pos, int32_t batch, int32_t n_new,
                                            float* k_tok_scale, float* v_tok_scale,
                                            float* v_scale_bound, void* stream) {
  if (!k_tok_scale || !v_tok_scale || !v_scale_bound) return ATLAS_ERR_INVALID_ARG;
  if (!aligned(k_tok_scale, 16) || !aligned(v_tok_scale, 16)) return ATLAS_ERR_INVALID_ARG;
  return append_impl(pool, k_new, v_new, dtype, block_table, max_blocks_per_seq, start_pos,
                     batch, n_new, k_tok_scale, v_tok_scale, v_scale_bound, stream);
}

atlas_status_t atlas_rope_fp8_kv_append(const atlas_kv_pool_t* pool, const void* qkv,
                                        int32_t num_q_heads, const float* cos_sin,
                                        int32_t max_pos, const int32_t* block_table,
                                        int32_t max_blocks_per_seq, const int32_t* start_pos,
                                        int32_t batch, int32_t n_new, void* q_out,
                                        void* stream) {
  if (!pool) return ATLAS_ERR_INVALID_ARG;
  if (batch < 0 || n_new < 0 || max_blocks_per_seq < 1 || num_q_heads < 1 || max_pos < 1)
    return ATLAS_ERR_INVALID_ARG;
  if (num_q_heads % pool->num_kv_heads != 0) return ATLAS_ERR_INVALID_ARG;
  if (batch == 0 || n_new == 0) return ATLAS_OK;
  if (!qkv || !cos_sin || !block_table || !start_pos || !q_out) return ATLAS_ERR_INVALID_ARG;
  if (!aligned(qkv, 16) || !aligned(cos_sin, 16) || !aligned(q_out, 16))
    return ATLAS_ERR_INVALID_ARG;
  atlas::RopeAppendParams p{};
  p.qkv = static_cast<const __nv_bfloat16*>(qkv);
  p.cos_sin = cos_sin;
  p.max_pos = max_pos;
  p.q_out = static_cast<__nv_bfloat16*>(q_out);
  p.k_pages = pool->k_pages;
  p.v_pages = pool->v_pages;
  p.k_scale = pool->k_scale;
  p.v_scale = pool->v_scale;
  p.block_table = block_table;
  p.start_pos = start_pos;
  p.err = reinterpret_cast<int32_t*>(pool->workspace);
  p.batch = batch;
  p.n_new = n_new;
  p.Hq = num_q_heads;
  p.Hkv = pool->num_kv_heads;
  p.D = pool->head_dim;
  p.ps = pool->page_size;
  p.num_pages = pool->num_pages;
  p.max_blocks = max_blocks_per_seq;
  cudaError_t e = atlas::launch_rope_append(p, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? ATLAS_OK : ATLAS_ERR_CUDA;
}

static atlas_status_t check_decode_shape(const atlas_kv_pool_t* pool, int32_t batch,
                                         int32_t num_q_heads, int32_t q_len,
                                         int32_t max_seq_len) {
  if (!pool) return ATLAS_ERR_INVALID_ARG;
  if (batch < 0 || batch > pool->max_batch) return ATLAS_ERR_INVALID_ARG;
  if (num_q_heads < 1 || num_q_heads % pool->num_kv_heads != 0) return ATLAS_ERR_INVALID_ARG;
  if (q_len < 1 || q_len > pool->max_q_len) return ATLAS_ERR_INVALID_ARG;
  if (max_seq_len < q_len) return ATLAS_ERR_INVALID_ARG;
  return ATLAS_OK;
}

atlas_status_t atlas_paged_gqa_decode_plan(const atlas_kv_pool_t* pool, int32_t batch,
                                           int32_t num_q_heads, int32_t q_len,
                                           int32_t max_seq_len, int32_t* plan, int32_t n) {
  atlas_status_t st = check_decode_shape(pool, batch, num_q_heads, q_len, max_seq_len);
  if (st != ATLAS_OK) return st;
  if (!plan || n < 0) return ATLAS_ERR_INVALID_ARG;
  const bool dev = device_present();
  const int sms = dev ? device_sm_count() : kDefaultSms;
  bool tc = false;
  const atlas::DecodeLaunch L =
      make_plan(pool, batch, num_q_heads, q_len, max_seq_len, sms, dev, &tc);
  long long spread = L.num_splits;  // grid partition: splits per segment
  if (!L.grid_mode) {  // balanced: most ranges a max-length segment can meet
    const long long seg_units = ((long long)max_seq_len + 31) / 32;
    spread = 1 + (seg_units - 1 + L.max_units - 1) / L.max_units;
    if (spread > L.grid) spread = L.grid;
  }
  const int32_t split = (!tc && pool->split_override > 0) ? pool->split_override : L.split_tokens;
  const int32_t f[ATLAS_PLAN_FIELDS] = {split, (int32_t)spread, tc ? 3 : L.grid_mode ? 1 : 2,
                                        L.rows_per_cta, L.row_blocks, 1,
                                        (int32_t)(L.grid > 0x7FFFFFFF ? 0x7FFFFFFF : L.grid)};
  for (int i = 0; i < n && i < ATLAS_PLAN_FIELDS; ++i) plan[i] = f[i];
  return ATLAS_OK;
}

}  // extern "C"

static atlas_status_t decode_impl(const atlas_kv_pool_t* pool, const void* q,
                                  const void* k_pages, const void* v_pages,
                                  const float* k_scale, const float* v_scale,
                                  const int32_t* block_table, int32_t max_blocks_per_seq,
                                  const int32_t* seq_lens, int32_t batch, int32_t num_q_heads,
                                  int32_t q_len, int32_t max_seq_len, float sm_scale, void* out,
                                  const void* k_new, const void* v_new, int32_t new_dtype,
                                  void* stream, const int32_t* cu_q = nullptr,
                                  const float* k_tok_scale = nullptr,
                                  const float* v_tok_scale = nullptr) {
  atlas_status_t st = check_decode_shape(pool, batch, num_q_heads, q_len, max_seq_len);
  if (st != ATLAS_OK) return st;
  if (max_blocks_per_seq < 1) return ATLAS_ERR_INVALID_ARG;
  if ((long long)max_seq_len > (long long)max_blocks_per_seq * pool->page_size)
    return ATLAS_ERR_INVALID_ARG;
  if (!(sm_scale == sm_scale) || isinf(sm_scale)) return ATLAS_ERR_INVALID_ARG;
  if (batch == 0) return ATLAS_OK;
  if (!q || !k_pages || !v_pages || !k_scale || !v_scale || !block_table || !seq_lens || !out)
    return ATLAS_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(out, 16) || !aligned(k_pages, 16) || !aligned(v_pages, 16))
    return ATLAS_ERR_INVALID_ARG;

  const int sms = device_sm_count();
  bool tc = false;
  atlas::DecodeLaunch L =
      make_plan(pool, batch, num_q_heads, q_len, max_seq_len, sms, true, &tc, cu_q != nullptr);
  if (k_tok_scale && !tc) {  // finer-grained scales: the tensor-core kernel only
    if (pool->head_dim != 128) return ATLAS_ERR_UNSUPPORTED;
    tc = true;
    L = atlas::plan_decode_tc(batch, num_q_heads, pool->num_kv_heads, q_len, max_seq_len, sms,
                              pool->split_override, pool->stages_override,
                              pool->waves_override > 0 ? pool->waves_override : 1);
  }
  const WsLayout ws = ws_layout(L, pool->head_dim);
  if (ws.total > pool->workspace_bytes) return ATLAS_ERR_WORKSPACE;
  if (L.grid > 0x7FFFFFFFLL) return ATLAS_ERR_UNSUPPORTED;

  atlas::DecodeParams p{};  // value-initialised: no fused append unless set
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.k_pages = static_cast<const uint8_t*>(k_pages);
  p.v_pages = static_cast<const uint8_t*>(v_pages);
  p.k_scale = k_scale;
  p.v_scale = v_scale;
  p.block_table = block_table;
  p.seq_lens = seq_lens;
  p.cu_q = cu_q;
  p.out = static_cast<__nv_bfloat16*>(out);
  uint8_t* wsp = pool->workspace;
  p.err = reinterpret_cast<int32_t*>(wsp);
  p.counters = reinterpret_cast<int32_t*>(wsp + ws.counters);
  p.part_lse = reinterpret_cast<float*>(wsp + ws.lse);
  p.part_o = reinterpret_cast<float*>(wsp + ws.o);
  p.B = batch;
  p.Hq = num_q_heads;
  p.Hkv = pool->num_kv_heads;
  p.G = num_q_heads / pool->num_kv_heads;
  p.q_len = q_len;
  p.D = pool->head_dim;
  p.ps = pool->page_size;
  p.num_pages = pool->num_pages;
  p.max_blocks = max_blocks_per_seq;
  p.max_seq_len = max_seq_len;
  p.row_blocks = L.row_blocks;
  p.max_units = L.max_units;
  p.max_portions = L.max_portions;
  p.grid_mode = L.grid_mode;
  p.num_splits = L.num_splits;
  p.split_tokens = L.split_tokens;
  const double scale = sm_scale > 0.f ? (double)sm_scale : 1.0 / sqrt((double)pool->head_dim);
  p.qk_scale_log2 = (float)(scale * 1.4426950408889634);  // log2(e)
  p.k_new = k_new;
  p.v_new = v_new;
  p.new_dtype = new_dtype;
  p.wait_limit_ns = pool->wait_limit_us > 0 ? 1000ull * pool->wait_limit_us
                                            : atlas::kDefaultWaitLimitNs;
  p.k_tok_scale = k_tok_scale;
  p.v_tok_scale = v_tok_scale;
  p.test_skip_unit = pool->test_skip_unit;
  cudaError_t e =
      tc ? atlas::launch_decode_tc(p, L.stages, L.grid, static_cast<cudaStream_t>(stream))
         : atlas::launch_decode_fp8(p, L.rows_per_warp, L.rbg, L.stages, L.grid,
                                    static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? ATLAS_OK : ATLAS_ERR_CUDA;
}


extern "C" {

atlas_status_t atlas_paged_gqa_decode(const atlas_kv_pool_t* pool, const void* q,
                                      const void* k_pages, const void* v_pages,
                                      const float* k_scale, const float* v_scale,
                                      const int32_t* block_table, int32_t max_blocks_per_seq,
                                      const int32_t* seq_lens, int32_t batch,
                                      int32_t num_q_heads, int32_t q_len, int32_t max_seq_len,
                                      float sm_scale, void* out, void* stream) {
  return decode_impl(pool, q, k_pages, v_pages, k_scale, v_scale, block_table,
                     max_blocks_per_seq, seq_lens, batch, num_q_heads, q_len, max_seq_len,
                     sm_scale, out, nullptr, nullptr, ATLAS_DTYPE_F32, stream);
}

atlas_status_t atlas_paged_gqa_decode_tokscale(const atlas_kv_pool_t* pool, const void* q,
                                               const float* k_tok_scale,
                                               const float* v_tok_scale,
                                               const float* v_scale_bound,
                                               const int32_t* block_table,
                                               int32_t max_blocks_per_seq,
                                               const int32_t* seq_lens, int32_t batch,
                                               int32_t num_q_heads, int32_t q_len,
                                               int32_t max_seq_len, float sm_scale, void* out,
                                               void* stream) {
  if (!pool) return ATLAS_ERR_INVALID_ARG;
  if (pool->head_dim != 128) return ATLAS_ERR_UNSUPPORTED;
  if (batch > 0 && (!k_tok_scale || !v_tok_scale || !v_scale_bound)) return ATLAS_ERR_INVALID_ARG;
  if (batch > 0 && (!aligned(k_tok_scale, 16) || !aligned(v_tok_scale, 16)))
    return ATLAS_ERR_INVALID_ARG;
  return decode_impl(pool, q, pool->k_pages, pool->v_pages, pool->k_scale, v_scale_bound,
                     block_table, max_blocks_per_seq, seq_lens, batch, num_q_heads, q_len,
                     max_seq_len, sm_scale, out, nullptr, nullptr, ATLAS_DTYPE_F32, stream,
                     nullptr, k_tok_scale, v_tok_scale);
}

atlas_status_t atlas_paged_gqa_decode_varlen(const atlas_kv_pool_t* pool, const void* q,
                                             const int32_t* cu_q_lens, const void* k_pages,
                                             const void* v_pages, const float* k_scale,
                                             const float* v_scale, const int32_t* block_table,
                                             int32_t max_blocks_per_seq, const int32_t* seq_lens,
                                             int32_t batch, int32_t num_q_heads,
                                             int32_t max_q_len, int32_t max_seq_len,
                                             float sm_scale, void* out, void* stream) {
  if (batch > 0 && !cu_q_lens) return ATLAS_ERR_INVALID_ARG;
  return decode_impl(pool, q, k_pages, v_pages, k_scale, v_scale, block_table,
                     max_blocks_per_seq, seq_lens, batch, num_q_heads, max_q_len, max_seq_len,
                     sm_scale, out, nullptr, nullptr, ATLAS_DTYPE_F32, stream, cu_q_lens);
}

atlas_status_t atlas_paged_gqa_append_decode(const atlas_kv_pool_t* pool, const void* k_new,
                                             const void* v_new, int32_t dtype, const void* q,
                                             const int32_t* block_table,
                                             int32_t max_blocks_per_seq, const int32_t* seq_lens,
                                             int32_t batch, int32_t num_q_heads, int32_t q_len,
                                             int32_t max_seq_len, float sm_scale, void* out,
                                             void* stream) {
  if (!pool) return ATLAS_ERR_INVALID_ARG;
  if (dtype != ATLAS_DTYPE_F32 && dtype != ATLAS_DTYPE_BF16) return ATLAS_ERR_INVALID_ARG;
  if (batch > 0 && (!k_new || !v_new)) return ATLAS_ERR_INVALID_ARG;
  if (batch > 0 && (!aligned(k_new, 16) || !aligned(v_new, 16))) return ATLAS_ERR_INVALID_ARG;
  return decode_impl(pool, q, pool->k_pages, pool->v_pages, pool->k_scale, pool->v_scale,
                     block_table, max_blocks_per_seq, seq_lens, batch, num_q_heads, q_len,
                     max_seq_len, sm_scale, out, k_new, v_new, dtype, stream);
}

atlas_status_t atlas_mtp_greedy_accept(const atlas_kv_pool_t* pool, const void* logits,
                                       int32_t dtype, int32_t batch, int32_t num_drafts,
                                       int32_t vocab, const int32_t* drafts, int32_t* targets,
                                       int32_t* n_accepted, int32_t* next_token, void* stream) {
  if (!pool) return ATLAS_ERR_INVALID_ARG;
  if (batch < 0 || batch > pool->max_batch || num_drafts < 0 || vocab < 1)
    return ATLAS_ERR_INVALID_ARG;
  if (dtype != ATLAS_DTYPE_F32 && dtype != ATLAS_DTYPE_BF16) return ATLAS_ERR_INVALID_ARG;
  if (batch == 0) return ATLAS_OK;
  if (!logits || !targets || !n_accepted || !next_token || (num_drafts > 0 && !drafts))
    return ATLAS_ERR_INVALID_ARG;
  if ((size_t)batch * sizeof(int32_t) > pool->counters_bytes) return ATLAS_ERR_WORKSPACE;
  int32_t* counters = reinterpret_cast<int32_t*>(pool->workspace + kAlign);
  cudaError_t e = atlas::launch_mtp_accept(logits, dtype, batch, num_drafts, vocab, drafts,
                                           targets, n_accepted, next_token, counters,
                                           static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? ATLAS_OK : ATLAS_ERR_CUDA;
}

atlas_status_t atlas_get_device_error(const atlas_kv_pool_t* pool, void* stream, int32_t* code) {
  if (!pool || !code) return ATLAS_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int32_t host = 0;
  if (cudaMemcpyAsync(&host, pool->workspace, sizeof(int32_t), cudaMemcpyDeviceToHost, s) !=
          cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess)
    return ATLAS_ERR_CUDA;
  // a call that stopped early (a timed-out wait) can leave completion counters
  // set: clear them with the error word
  if (host != 0 && (cudaMemsetAsync(pool->workspace, 0, kAlign + pool->counters_bytes, s) !=
                        cudaSuccess ||
                    cudaStreamSynchronize(s) != cudaSuccess))
    return ATLAS_ERR_CUDA;
  *code = host;
  return host == 0 ? ATLAS_OK : ATLAS_ERR_DEVICE_CHECK;
}

}  // extern "C"
