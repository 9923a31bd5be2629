// C ABI of the window-step library: argument checks, descriptor bookkeeping, launches.
// The operations and their sources are documented in include/dp.h.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <vector>

#include "dp.h"
#include "dp_internal.h"

namespace {

thread_local char g_detail[512] = "";
// Stage profiling of dp_window_step and dp_sublayer_step (per thread): up to kProfEvents
// events per recorded step (stage boundaries), nst[i] stages in step i.
constexpr int kProfEvents = 6;
struct Profile {
  std::vector<cudaEvent_t> ev;
  std::vector<int> nst;
  int32_t max_steps = 0;
  int32_t count = 0;
  bool active = false;
};
thread_local Profile g_prof;

cudaEvent_t prof_event(int stage) {
  if (!g_prof.active || g_prof.count >= g_prof.max_steps) return nullptr;
  return g_prof.ev[kProfEvents * g_prof.count + stage];
}

// A step that recorded its events counts once it has recorded the last one.
void prof_step_done(cudaEvent_t last, int n_stages) {
  if (!last) return;
  g_prof.nst[g_prof.count] = n_stages;
  g_prof.count += 1;
}

cudaError_t record(cudaEvent_t ev, cudaStream_t s) { return ev ? cudaEventRecord(ev, s) : cudaSuccess; }

dp_status fail(dp_status s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_detail, sizeof(g_detail), fmt, ap);
  va_end(ap);
  return s;
}

dp_status cuda_fail(cudaError_t e, const char* what) {
  return fail(DP_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int elem_bytes(dp_dtype dt) { return dt == DP_F32 ? 4 : 2; }

bool dtype_ok(dp_dtype dt) { return dt == DP_BF16 || dt == DP_F16 || dt == DP_F32; }

// Element type of the modulated features (k', v', cache) for a window of type dt.
dp_dtype feature_dtype(dp_dtype dt) { return dt == DP_F32 ? DP_F32 : DP_F16; }

bool modulate_pair_ok(dp_dtype x, dp_dtype y) {
  return (x == DP_BF16 && (y == DP_BF16 || y == DP_F16)) || (x == DP_F16 && y == DP_F16) ||
         (x == DP_F32 && y == DP_F32);
}

// Row pitch must be a whole number of 16-byte vectors.
bool hidden_ok(int32_t hidden, dp_dtype dt) {
  return hidden > 0 && (static_cast<int64_t>(hidden) * elem_bytes(dt)) % 16 == 0;
}

dp_status check_blocks(const dp_blocks* blk, int64_t n_rows, int32_t hidden) {
  if (!blk) return fail(DP_ERR_INVALID_ARG, "block table is NULL");
  if (blk->n_blocks < 1 || blk->n_blocks > DP_MAX_BLOCKS)
    return fail(DP_ERR_INVALID_ARG, "n_blocks %d outside [1, %d]", blk->n_blocks, DP_MAX_BLOCKS);
  if (blk->hidden != hidden) return fail(DP_ERR_INVALID_ARG, "block table hidden %d != %d", blk->hidden, hidden);
  if (blk->row_offset[0] != 0) return fail(DP_ERR_INVALID_ARG, "row_offset[0] must be 0");
  for (int b = 0; b < blk->n_blocks; ++b) {
    if (blk->row_offset[b + 1] < blk->row_offset[b]) return fail(DP_ERR_INVALID_ARG, "row_offset decreases at %d", b);
    if (!blk->mod[b] || !aligned16(blk->mod[b])) return fail(DP_ERR_INVALID_ARG, "mod[%d] NULL or misaligned", b);
  }
  if (blk->row_offset[blk->n_blocks] != n_rows)
    return fail(DP_ERR_INVALID_ARG, "row_offset[n_blocks] = %d != rows %lld", blk->row_offset[blk->n_blocks],
                static_cast<long long>(n_rows));
  return DP_OK;
}

dp::BlockTable to_table(const dp_blocks* blk) {
  dp::BlockTable t;
  memset(&t, 0, sizeof(t));
  t.n_blocks = blk->n_blocks;
  for (int b = 0; b <= blk->n_blocks; ++b) t.row_offset[b] = blk->row_offset[b];
  for (int b = blk->n_blocks + 1; b <= DP_MAX_BLOCKS; ++b) t.row_offset[b] = blk->row_offset[blk->n_blocks];
  for (int b = 0; b < blk->n_blocks; ++b) t.mod[b] = blk->mod[b];
  for (int b = blk->n_blocks; b < DP_MAX_BLOCKS; ++b) t.mod[b] = blk->mod[0];
  return t;
}

constexpr int kMaxDevices = 64;
uint32_t* g_status_ptr[kMaxDevices] = {};
std::mutex g_status_mu;

}  // namespace

// The device status word bounded waits write to (one per device that loads the library).
__device__ uint32_t dp_status_word;

namespace {

dp_status status_ptr(uint32_t** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(DP_ERR_UNSUPPORTED, "device ordinal %d", dev);
  std::lock_guard<std::mutex> lk(g_status_mu);
  if (!g_status_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, dp_status_word);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(status word)");
    g_status_ptr[dev] = static_cast<uint32_t*>(p);
  }
  *out = g_status_ptr[dev];
  return DP_OK;
}

int64_t cache_read_slot(const dp_kvcache* c) {
  return c->n_advances > 0 ? (c->n_advances - 1) % c->n_slots : 0;
}

dp_status check_cache(const dp_kvcache* c, int32_t hidden, dp_dtype dt) {
  if (!c) return fail(DP_ERR_INVALID_ARG, "cache is NULL");
  if (!c->k || !c->v || !aligned16(c->k) || !aligned16(c->v))
    return fail(DP_ERR_INVALID_ARG, "cache k/v NULL or misaligned");
  if (c->hidden != hidden || c->dtype != dt) return fail(DP_ERR_INVALID_ARG, "cache hidden/dtype mismatch");
  if (c->n_slots < 1 || c->n_slots > DP_MAX_SLOTS) return fail(DP_ERR_INVALID_ARG, "cache n_slots %d", c->n_slots);
  if (c->capacity < 0 || c->n_advances < 0) return fail(DP_ERR_INVALID_ARG, "cache capacity/n_advances negative");
  if (c->capacity * c->n_slots > INT32_MAX) return fail(DP_ERR_CAPACITY, "cache ring rows exceed 2^31 - 1");
  for (int s = 0; s < c->n_slots; ++s)
    if (c->len[s] < 0 || c->len[s] > c->capacity)
      return fail(DP_ERR_CAPACITY, "cache len[%d] = %lld outside [0, capacity]", s, static_cast<long long>(c->len[s]));
  return DP_OK;
}

dp_status check_queue(const dp_queue* q, int32_t hidden, dp_dtype dt) {
  if (!q->latent || !aligned16(q->latent)) return fail(DP_ERR_INVALID_ARG, "queue latent NULL or misaligned");
  if (q->hidden != hidden || q->dtype != dt) return fail(DP_ERR_INVALID_ARG, "queue hidden/dtype mismatch");
  if (q->n_slots < 1 || q->n_slots > DP_MAX_SLOTS) return fail(DP_ERR_INVALID_ARG, "queue n_slots %d", q->n_slots);
  if (q->count < 0 || q->count > q->n_slots || q->head < 0 || q->head >= q->n_slots || q->slot_rows <= 0)
    return fail(DP_ERR_INVALID_ARG, "queue head/count/slot_rows inconsistent");
  return DP_OK;
}

// Physical slot p of the mirrored ring: copies land at slots p and p + n_slots.
char* queue_slot(const dp_queue* q, int32_t p) {
  const int64_t pitch = q->slot_rows * q->hidden * elem_bytes(q->dtype);
  return static_cast<char*>(q->latent) + static_cast<int64_t>(p) * pitch;
}

dp_status check_push(const dp_queue* q, int32_t count_after_pop, const void* noise, int64_t rows) {
  if (!noise || !aligned16(noise)) return fail(DP_ERR_INVALID_ARG, "push noise NULL or misaligned");
  if (rows <= 0) return fail(DP_ERR_INVALID_ARG, "push rows %lld", static_cast<long long>(rows));
  if (rows > q->slot_rows) return fail(DP_ERR_CAPACITY, "push rows %lld > slot_rows", static_cast<long long>(rows));
  if (count_after_pop >= q->n_slots) return fail(DP_ERR_CAPACITY, "queue full (%d blocks)", q->n_slots);
  if (count_after_pop > 0) {
    // the tail is the block at logical position count_after_pop - 1 (after any pop)
    const int shift = q->count - count_after_pop;  // 1 if the head was popped
    const int32_t tail_rows = q->rows[count_after_pop - 1 + shift];
    if (tail_rows < q->slot_rows) return fail(DP_ERR_INVALID_ARG, "no push may follow a short final block");
  }
  return DP_OK;
}

void apply_pop(dp_queue* q) {
  for (int i = 1; i < q->count; ++i) {
    q->rows[i - 1] = q->rows[i];
    q->evals[i - 1] = q->evals[i];
  }
  q->count -= 1;
  q->rows[q->count] = 0;
  q->evals[q->count] = 0;
  q->head = (q->head + 1) % q->n_slots;
  q->n_popped += 1;
}

int32_t apply_push(dp_queue* q, int64_t rows) {
  const int32_t p = (q->head + q->count) % q->n_slots;
  q->rows[q->count] = static_cast<int32_t>(rows);
  q->evals[q->count] = 0;
  q->count += 1;
  q->n_pushed += 1;
  return p;
}

}  // namespace

namespace dp {
dp_status set_error(dp_status s, const char* msg) { return fail(s, "%s", msg); }
}  // namespace dp

extern "C" {

int32_t dp_version(void) { return 100; }

const char* dp_status_string(dp_status s) {
  switch (s) {
    case DP_OK: return "DP_OK";
    case DP_ERR_INVALID_ARG: return "DP_ERR_INVALID_ARG";
    case DP_ERR_UNSUPPORTED: return "DP_ERR_UNSUPPORTED";
    case DP_ERR_CUDA: return "DP_ERR_CUDA";
    case DP_ERR_CAPACITY: return "DP_ERR_CAPACITY";
    case DP_ERR_TIMEOUT: return "DP_ERR_TIMEOUT";
    case DP_ERR_EMPTY: return "DP_ERR_EMPTY";
  }
  return "DP_ERR_UNKNOWN";
}

const char* dp_last_error_detail(void) { return g_detail; }

dp_status dp_profile_begin(int32_t max_steps) {
  if (max_steps < 1) return fail(DP_ERR_INVALID_ARG, "max_steps %d", max_steps);
  if (g_prof.active) return fail(DP_ERR_INVALID_ARG, "profiling already active");
  g_prof.ev.assign(static_cast<size_t>(kProfEvents) * max_steps, nullptr);
  g_prof.nst.assign(static_cast<size_t>(max_steps), 0);
  for (auto& e : g_prof.ev) {
    cudaError_t r = cudaEventCreate(&e);
    if (r != cudaSuccess) {
      for (auto& x : g_prof.ev)
        if (x) cudaEventDestroy(x);
      g_prof.ev.clear();
      return cuda_fail(r, "cudaEventCreate");
    }
  }
  g_prof.max_steps = max_steps;
  g_prof.count = 0;
  g_prof.active = true;
  return DP_OK;
}

namespace {

// Per-stage sums (ms) over the recorded steps, then the events are released.
dp_status profile_collect(double (&sum)[kProfEvents - 1], int* n_stages) {
  if (!g_prof.active) return fail(DP_ERR_INVALID_ARG, "profiling not active");
  for (double& x : sum) x = 0.0;
  *n_stages = 0;
  dp_status st = DP_OK;
  if (g_prof.count > 0) {
    const int last = g_prof.count - 1;
    cudaError_t r = cudaEventSynchronize(g_prof.ev[kProfEvents * last + g_prof.nst[last]]);
    for (int i = 0; r == cudaSuccess && i < g_prof.count; ++i) {
      *n_stages = g_prof.nst[i] > *n_stages ? g_prof.nst[i] : *n_stages;
      for (int k = 0; r == cudaSuccess && k < g_prof.nst[i]; ++k) {
        float ms = 0.0f;
        r = cudaEventElapsedTime(&ms, g_prof.ev[kProfEvents * i + k], g_prof.ev[kProfEvents * i + k + 1]);
        sum[k] += ms;
      }
    }
    if (r != cudaSuccess) st = cuda_fail(r, "event timing");
  }
  for (auto& e : g_prof.ev) cudaEventDestroy(e);
  g_prof.ev.clear();
  g_prof.nst.clear();
  g_prof.active = false;
  return st;
}

}  // namespace

dp_status dp_profile_end(float* ms_modulate, float* ms_attention, float* ms_advance, int32_t* steps) {
  if (!g_prof.active) return fail(DP_ERR_INVALID_ARG, "profiling not active");
  double sum[kProfEvents - 1];
  int n_stages = 0;
  const int32_t count = g_prof.count;
  dp_status st = profile_collect(sum, &n_stages);
  if (ms_modulate) *ms_modulate = static_cast<float>(sum[0]);
  if (ms_attention) *ms_attention = static_cast<float>(sum[1]);
  if (ms_advance) *ms_advance = static_cast<float>(sum[2]);
  if (steps) *steps = count;
  return st;
}

dp_status dp_profile_end_stages(float* ms, int32_t max_stages, int32_t* n_stages, int32_t* steps) {
  if (!g_prof.active) return fail(DP_ERR_INVALID_ARG, "profiling not active");
  double sum[kProfEvents - 1];
  int ns = 0;
  const int32_t count = g_prof.count;
  dp_status st = profile_collect(sum, &ns);
  if (ms)
    for (int k = 0; k < max_stages && k < kProfEvents - 1; ++k) ms[k] = static_cast<float>(sum[k]);
  if (n_stages) *n_stages = ns;
  if (steps) *steps = count;
  return st;
}

dp_status dp_set_device(int32_t ordinal) {
  cudaError_t e = cudaSetDevice(ordinal);
  if (e != cudaSuccess) return cuda_fail(e, "cudaSetDevice");
  return DP_OK;
}

dp_status dp_device_status(void* stream) {
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  uint32_t word = 0;
  e = cudaMemcpyFromSymbol(&word, dp_status_word, sizeof(word));
  if (e != cudaSuccess) return cuda_fail(e, "read status word");
  if (word) {
    const uint32_t zero = 0;
    e = cudaMemcpyToSymbol(dp_status_word, &zero, sizeof(zero));
    if (e != cudaSuccess) return cuda_fail(e, "clear status word");
    return fail(DP_ERR_TIMEOUT, "device wait gave up (status word 0x%x)", word);
  }
  return DP_OK;
}

dp_status dp_blocks_from_table(dp_blocks* out, const float* table, int32_t table_rows, int32_t hidden,
                               const int32_t* timesteps, const int32_t* block_rows, int32_t n_blocks) {
  if (!out || !table || !timesteps || !block_rows) return fail(DP_ERR_INVALID_ARG, "NULL argument");
  if (n_blocks < 1 || n_blocks > DP_MAX_BLOCKS) return fail(DP_ERR_INVALID_ARG, "n_blocks %d", n_blocks);
  if (hidden <= 0 || hidden % 4) return fail(DP_ERR_INVALID_ARG, "hidden %d", hidden);
  if (!aligned16(table)) return fail(DP_ERR_INVALID_ARG, "table misaligned");
  dp_blocks b;
  memset(&b, 0, sizeof(b));
  b.n_blocks = n_blocks;
  b.hidden = hidden;
  int64_t off = 0;
  for (int i = 0; i < n_blocks; ++i) {
    if (timesteps[i] < 0 || timesteps[i] >= table_rows)
      return fail(DP_ERR_INVALID_ARG, "timestep %d outside [0, %d)", timesteps[i], table_rows);
    if (block_rows[i] < 0) return fail(DP_ERR_INVALID_ARG, "block_rows[%d] negative", i);
    b.row_offset[i] = static_cast<int32_t>(off);
    off += block_rows[i];
    if (off > INT32_MAX) return fail(DP_ERR_INVALID_ARG, "window rows overflow");
    b.mod[i] = table + static_cast<int64_t>(timesteps[i]) * 3 * hidden;
  }
  b.row_offset[n_blocks] = static_cast<int32_t>(off);
  *out = b;
  return DP_OK;
}

dp_status dp_queue_blocks(const dp_queue* q, const float* table, int32_t table_rows, const int32_t* tau, int32_t n_tau,
                          dp_blocks* out, const void** window, int64_t* n_win) {
  if (!q || !table || !tau || !out || !window || !n_win) return fail(DP_ERR_INVALID_ARG, "NULL argument");
  dp_status st = check_queue(q, q->hidden, q->dtype);
  if (st != DP_OK) return st;
  if (q->count == 0) return fail(DP_ERR_EMPTY, "queue is empty");
  int32_t ts[DP_MAX_SLOTS];
  for (int i = 0; i < q->count; ++i) {
    if (q->evals[i] < 0 || q->evals[i] >= n_tau)
      return fail(DP_ERR_INVALID_ARG, "block %d has had %d evaluations of %d", i, q->evals[i], n_tau);
    ts[i] = tau[q->evals[i]];
  }
  st = dp_blocks_from_table(out, table, table_rows, q->hidden, ts, q->rows, q->count);
  if (st != DP_OK) return st;
  *window = queue_slot(q, q->head);
  *n_win = out->row_offset[q->count];
  return DP_OK;
}

dp_status dp_adaln_modulate(const void* x, void* y, int64_t n_rows, const dp_blocks* blk, dp_dtype x_dt,
                            dp_dtype y_dt, void* stream) {
  if (!dtype_ok(x_dt) || !dtype_ok(y_dt)) return fail(DP_ERR_INVALID_ARG, "dtype");
  if (!modulate_pair_ok(x_dt, y_dt)) return fail(DP_ERR_UNSUPPORTED, "modulation %d -> %d", x_dt, y_dt);
  const dp_dtype dt = x_dt;
  if (!x || !y || !aligned16(x) || !aligned16(y)) return fail(DP_ERR_INVALID_ARG, "x/y NULL or misaligned");
  if (n_rows <= 0) return fail(DP_ERR_INVALID_ARG, "n_rows %lld", static_cast<long long>(n_rows));
  if (!blk) return fail(DP_ERR_INVALID_ARG, "block table is NULL");
  if (!hidden_ok(blk->hidden, dt)) return fail(DP_ERR_INVALID_ARG, "hidden %d not a whole number of 16-byte vectors", blk->hidden);
  dp_status st = check_blocks(blk, n_rows, blk->hidden);
  if (st != DP_OK) return st;
  const dp::BlockTable t = to_table(blk);
  const void* src[1] = {x};
  void* dst[1] = {y};
  cudaError_t e = dp::launch_modulate(src, dst, 1, n_rows, blk->hidden, t, x_dt, y_dt, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "modulate launch");
  return DP_OK;
}

namespace {

dp_status check_attention(const void* q, const void* k, const void* v, int64_t n_win, const void* ck, const void* cv,
                          int64_t cache_len, const void* residual, void* out, int32_t n_heads, int32_t head_dim,
                          const dp_blocks* blk, dp_dtype dt, dp_dtype ft) {
  if (!dtype_ok(dt) || !dtype_ok(ft)) return fail(DP_ERR_INVALID_ARG, "dtype");
  const bool tc = dt == DP_BF16 && (ft == DP_F16 || ft == DP_BF16);
  if (!tc && !(dt == DP_F32 && ft == DP_F32))
    return fail(DP_ERR_UNSUPPORTED, "window/feature dtypes %d/%d (bf16/f16, bf16/bf16 or f32/f32)", dt, ft);
  if (!q || !k || !v || !out) return fail(DP_ERR_INVALID_ARG, "q/k/v/out NULL");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || (residual && !aligned16(residual)))
    return fail(DP_ERR_INVALID_ARG, "pointer not 16-byte aligned");
  if (n_win <= 0 || n_win > INT32_MAX) return fail(DP_ERR_INVALID_ARG, "n_win %lld", static_cast<long long>(n_win));
  if (cache_len < 0 || cache_len > INT32_MAX) return fail(DP_ERR_INVALID_ARG, "cache_len %lld", static_cast<long long>(cache_len));
  if (cache_len > 0 && (!ck || !cv || !aligned16(ck) || !aligned16(cv)))
    return fail(DP_ERR_INVALID_ARG, "cache k/v NULL or misaligned");
  if (n_heads <= 0 || head_dim <= 0) return fail(DP_ERR_INVALID_ARG, "n_heads/head_dim");
  const int64_t hidden = static_cast<int64_t>(n_heads) * head_dim;
  if (hidden > INT32_MAX || !hidden_ok(static_cast<int32_t>(hidden), dt)) return fail(DP_ERR_INVALID_ARG, "hidden");
  if (tc && head_dim != 64 && head_dim != 128)
    return fail(DP_ERR_UNSUPPORTED, "bf16 head_dim %d (64 or 128 supported)", head_dim);
  if (dt == DP_F32 && head_dim != 4 && head_dim != 8 && head_dim != 16 && head_dim != 32 && head_dim != 64 &&
      head_dim != 128)
    return fail(DP_ERR_UNSUPPORTED, "f32 head_dim %d (4, 8, 16, 32, 64 or 128 supported)", head_dim);
  if (out == q || out == k || out == v || (residual && out == residual) || (cache_len > 0 && (out == ck || out == cv)))
    return fail(DP_ERR_INVALID_ARG, "out aliases an input");
  return check_blocks(blk, n_win, static_cast<int32_t>(hidden));
}

// A single cache segment: rows [0, cache_len) of cache_k / cache_v.
dp::CacheSegs one_segment(int64_t cache_len) {
  dp::CacheSegs g;
  memset(&g, 0, sizeof(g));
  g.n = cache_len > 0 ? 1 : 0;
  g.len[0] = static_cast<int32_t>(cache_len);
  return g;
}

// The segments a step reads from the cache ring: the most recently written slot, or with
// DP_STEP_CACHE_ALL_SLOTS every slot that holds rows, oldest first.  Rows are counted from
// the ring's base (slot s starts at row s * capacity).
dp::CacheSegs ring_segments(const dp_kvcache* c, uint32_t flags, int64_t* total) {
  dp::CacheSegs g;
  memset(&g, 0, sizeof(g));
  *total = 0;
  if (flags & DP_STEP_CACHE_ALL_SLOTS) {
    for (int i = 0; i < c->n_slots; ++i) {
      const int64_t slot = (c->n_advances + i) % c->n_slots;  // oldest first
      if (c->len[slot] <= 0) continue;
      g.row[g.n] = static_cast<int32_t>(slot * c->capacity);
      g.len[g.n] = static_cast<int32_t>(c->len[slot]);
      *total += c->len[slot];
      g.n += 1;
    }
  } else {
    const int64_t slot = cache_read_slot(c);
    if (c->len[slot] > 0) {
      g.n = 1;
      g.row[0] = static_cast<int32_t>(slot * c->capacity);
      g.len[0] = static_cast<int32_t>(c->len[slot]);
      *total = c->len[slot];
    }
  }
  return g;
}

dp_status run_attention(const void* q, const void* k, const void* v, int64_t n_win, const void* ck, const void* cv,
                        const dp::CacheSegs& segs, int64_t cache_rows, const void* residual, void* out,
                        int32_t n_heads, int32_t head_dim, float softmax_scale, const dp_blocks* blk, uint32_t flags,
                        dp_dtype dt, dp_dtype ft, cudaStream_t s) {
  dp::AttnArgs a;
  a.q = q;
  a.k = k;
  a.v = v;
  a.cache_k = ck;
  a.cache_v = cv;
  a.residual = residual;
  a.out = out;
  a.n_win = n_win;
  a.cache_len = 0;
  for (int i = 0; i < segs.n; ++i) a.cache_len += segs.len[i];
  a.cache_rows = cache_rows;
  a.segs = segs;
  a.n_heads = n_heads;
  a.head_dim = head_dim;
  a.hidden = n_heads * head_dim;
  a.softmax_scale = softmax_scale > 0.0f ? softmax_scale : 1.0f / sqrtf(static_cast<float>(head_dim));
  a.flags = flags;
  a.bt = to_table(blk);
  dp_status st = status_ptr(&a.status);
  if (st != DP_OK) return st;
  cudaError_t e = dt == DP_BF16 ? dp::launch_attention_tc(a, ft == DP_F16, s) : dp::launch_attention_f32(a, s);
  if (e != cudaSuccess) return cuda_fail(e, "attention launch");
  return DP_OK;
}

}  // namespace

dp_status dp_window_attention(const void* q, const void* k, const void* v, int64_t n_win, const void* cache_k,
                              const void* cache_v, int64_t cache_len, const void* residual, void* out,
                              int32_t n_heads, int32_t head_dim, float softmax_scale, const dp_blocks* blk,
                              uint32_t flags, dp_dtype dt, dp_dtype feat_dt, void* stream) {
  dp_status st =
      check_attention(q, k, v, n_win, cache_k, cache_v, cache_len, residual, out, n_heads, head_dim, blk, dt, feat_dt);
  if (st != DP_OK) return st;
  return run_attention(q, k, v, n_win, cache_k, cache_v, one_segment(cache_len), cache_len, residual, out, n_heads,
                       head_dim, softmax_scale, blk, flags, dt, feat_dt, static_cast<cudaStream_t>(stream));
}

dp_status dp_kvcache_advance(dp_kvcache* c, const void* k_exit, const void* v_exit, int64_t n_exit, void* stream) {
  if (!c) return fail(DP_ERR_INVALID_ARG, "cache is NULL");
  dp_status st = check_cache(c, c->hidden, c->dtype);
  if (st != DP_OK) return st;
  if (!hidden_ok(c->hidden, c->dtype)) return fail(DP_ERR_INVALID_ARG, "hidden");
  if (n_exit < 0) return fail(DP_ERR_INVALID_ARG, "n_exit negative");
  if (n_exit > c->capacity)
    return fail(DP_ERR_CAPACITY, "exiting block of %lld rows > cache capacity %lld", static_cast<long long>(n_exit),
                static_cast<long long>(c->capacity));
  if (n_exit > 0 && (!k_exit || !v_exit || !aligned16(k_exit) || !aligned16(v_exit)))
    return fail(DP_ERR_INVALID_ARG, "k_exit/v_exit NULL or misaligned");
  const int64_t row_bytes = static_cast<int64_t>(c->hidden) * elem_bytes(c->dtype);
  const int64_t slot = c->n_advances % c->n_slots;
  dp::CopySeg segs[2] = {
      {k_exit, static_cast<char*>(c->k) + slot * c->capacity * row_bytes, n_exit * row_bytes},
      {v_exit, static_cast<char*>(c->v) + slot * c->capacity * row_bytes, n_exit * row_bytes}};
  cudaError_t e = dp::launch_copy(segs, 2, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "advance copy");
  c->len[slot] = n_exit;
  c->n_advances += 1;
  return DP_OK;
}

dp_status dp_queue_push(dp_queue* q, const void* noise, int64_t rows, void* stream) {
  if (!q) return fail(DP_ERR_INVALID_ARG, "queue is NULL");
  dp_status st = check_queue(q, q->hidden, q->dtype);
  if (st != DP_OK) return st;
  st = check_push(q, q->count, noise, rows);
  if (st != DP_OK) return st;
  const int64_t bytes = rows * q->hidden * elem_bytes(q->dtype);
  const int32_t p = (q->head + q->count) % q->n_slots;
  dp::CopySeg segs[2] = {{noise, queue_slot(q, p), bytes}, {noise, queue_slot(q, p + q->n_slots), bytes}};
  cudaError_t e = dp::launch_copy(segs, 2, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "push copy");
  apply_push(q, rows);
  return DP_OK;
}

dp_status dp_queue_push_frames(dp_queue* q, const void* pool, int32_t pool_frames, int64_t frame_rows,
                               const int32_t* frame_idx, int32_t n_frames, void* stream) {
  if (!q) return fail(DP_ERR_INVALID_ARG, "queue is NULL");
  dp_status st = check_queue(q, q->hidden, q->dtype);
  if (st != DP_OK) return st;
  if (!frame_idx) return fail(DP_ERR_INVALID_ARG, "frame_idx is NULL");
  if (n_frames < 1 || n_frames > dp::kMaxGatherFrames)
    return fail(DP_ERR_UNSUPPORTED, "n_frames %d outside [1, %d]", n_frames, dp::kMaxGatherFrames);
  if (pool_frames < 1 || frame_rows < 1) return fail(DP_ERR_INVALID_ARG, "pool_frames/frame_rows");
  for (int i = 0; i < n_frames; ++i)
    if (frame_idx[i] < 0 || frame_idx[i] >= pool_frames)
      return fail(DP_ERR_INVALID_ARG, "frame_idx[%d] = %d outside [0, %d)", i, frame_idx[i], pool_frames);
  const int64_t rows = frame_rows * n_frames;
  st = check_push(q, q->count, pool, rows);
  if (st != DP_OK) return st;
  const int64_t frame_bytes = frame_rows * q->hidden * elem_bytes(q->dtype);
  if (frame_bytes % 16 || frame_bytes / 16 > UINT32_MAX) return fail(DP_ERR_INVALID_ARG, "frame size");
  const int32_t p = (q->head + q->count) % q->n_slots;
  dp::FrameGather g;
  memset(&g, 0, sizeof(g));
  g.pool = static_cast<const uint4*>(pool);
  g.dst0 = static_cast<uint4*>(static_cast<void*>(queue_slot(q, p)));
  g.dst1 = static_cast<uint4*>(static_cast<void*>(queue_slot(q, p + q->n_slots)));
  g.vec_per_frame = static_cast<uint32_t>(frame_bytes / 16);
  g.n_frames = n_frames;
  for (int i = 0; i < n_frames; ++i) g.idx[i] = frame_idx[i];
  cudaError_t e = dp::launch_gather_frames(g, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "frame gather");
  apply_push(q, rows);
  return DP_OK;
}

dp_status dp_queue_pop(dp_queue* q) {
  if (!q) return fail(DP_ERR_INVALID_ARG, "queue is NULL");
  dp_status st = check_queue(q, q->hidden, q->dtype);
  if (st != DP_OK) return st;
  if (q->count == 0) return fail(DP_ERR_EMPTY, "queue is empty");
  apply_pop(q);
  return DP_OK;
}

dp_status dp_window_step(const void* q, const void* k, const void* v, int64_t n_win, const dp_blocks* blk,
                         dp_kvcache* cache, void* kv_work, const void* residual, void* out, int32_t n_heads,
                         int32_t head_dim, uint32_t flags, dp_queue* queue, const void* push_noise, int64_t push_rows,
                         dp_dtype dt, void* stream) {
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (!cache) return fail(DP_ERR_INVALID_ARG, "cache is NULL");
  const int64_t hidden64 = static_cast<int64_t>(n_heads) * head_dim;
  if (n_heads <= 0 || head_dim <= 0 || hidden64 > INT32_MAX) return fail(DP_ERR_INVALID_ARG, "n_heads/head_dim");
  const int32_t hidden = static_cast<int32_t>(hidden64);
  if (!dtype_ok(dt)) return fail(DP_ERR_INVALID_ARG, "dtype");
  const dp_dtype ft = feature_dtype(dt);
  dp_status st = check_cache(cache, hidden, ft);
  if (st != DP_OK) return st;
  if (!kv_work || !aligned16(kv_work)) return fail(DP_ERR_INVALID_ARG, "kv_work NULL or misaligned");
  const int64_t row_bytes = hidden64 * elem_bytes(ft);     // features: k', v', cache
  const int64_t in_row_bytes = hidden64 * elem_bytes(dt);  // window inputs and the latent queue
  int64_t cache_len = 0;
  const dp::CacheSegs cseg = ring_segments(cache, flags, &cache_len);
  const char* ck = static_cast<const char*>(cache->k);
  const char* cv = static_cast<const char*>(cache->v);
  const int64_t cache_rows = static_cast<int64_t>(cache->n_slots) * cache->capacity;
  char* kp = static_cast<char*>(kv_work);
  char* vp = kp + n_win * row_bytes;
  st = check_attention(q, kp, vp, n_win, ck, cv, cache_len, residual, out, n_heads, head_dim, blk, dt, ft);
  if (st != DP_OK) return st;
  if (!k || !v || !aligned16(k) || !aligned16(v)) return fail(DP_ERR_INVALID_ARG, "k/v NULL or misaligned");
  if (out == kv_work) return fail(DP_ERR_INVALID_ARG, "out aliases kv_work");
  const bool pop = (flags & DP_STEP_POP) != 0;
  const int64_t n_exit = blk->row_offset[1];
  if (pop && n_exit > cache->capacity)
    return fail(DP_ERR_CAPACITY, "head block of %lld rows > cache capacity", static_cast<long long>(n_exit));
  if (queue) {
    st = check_queue(queue, hidden, dt);
    if (st != DP_OK) return st;
    if (pop && queue->count == 0) return fail(DP_ERR_EMPTY, "pop from an empty queue");
  }
  if (push_noise) {
    if (!queue) return fail(DP_ERR_INVALID_ARG, "push needs a queue");
    st = check_push(queue, queue->count - (pop ? 1 : 0), push_noise, push_rows);
    if (st != DP_OK) return st;
  }

  // A1: k' and v' of the window (one launch, two segments)
  const dp::BlockTable t = to_table(blk);
  const void* src[2] = {k, v};
  void* dst[2] = {kp, vp};
  cudaEvent_t ev0 = prof_event(0), ev1 = prof_event(1), ev2 = prof_event(2), ev3 = prof_event(3);
  cudaError_t e = record(ev0, s);
  if (e == cudaSuccess) e = dp::launch_modulate(src, dst, 2, n_win, hidden, t, dt, ft, s);
  if (e == cudaSuccess) e = record(ev1, s);
  if (e != cudaSuccess) return cuda_fail(e, "modulate launch");
  // A2: attention with the Q prologue and gate epilogue
  st = run_attention(q, kp, vp, n_win, ck, cv, cseg, cache_rows, residual, out, n_heads, head_dim, 0.0f, blk,
                     DP_MOD_Q | DP_GATE_OUT, dt, ft, s);
  if (st != DP_OK) return st;
  e = record(ev2, s);
  if (e != cudaSuccess) return cuda_fail(e, "event record");
  // A3: pop (head block's k'/v' -> cache ring) and push (noise -> latent ring), one launch.
  // Descriptors change only after the launch has been accepted.
  dp::CopySeg segs[dp::kMaxCopySegs];
  int nseg = 0;
  const int64_t wslot = cache->n_advances % cache->n_slots;
  if (pop) {
    segs[nseg++] = {kp, static_cast<char*>(cache->k) + wslot * cache->capacity * row_bytes, n_exit * row_bytes};
    segs[nseg++] = {vp, static_cast<char*>(cache->v) + wslot * cache->capacity * row_bytes, n_exit * row_bytes};
  }
  if (push_noise) {
    const int32_t head_after = (queue->head + ((pop && queue) ? 1 : 0)) % queue->n_slots;
    const int32_t count_after = queue->count - (pop ? 1 : 0);
    const int32_t p = (head_after + count_after) % queue->n_slots;
    const int64_t bytes = push_rows * in_row_bytes;
    segs[nseg++] = {push_noise, queue_slot(queue, p), bytes};
    segs[nseg++] = {push_noise, queue_slot(queue, p + queue->n_slots), bytes};
  }
  if (nseg) {
    e = dp::launch_copy(segs, nseg, s);
    if (e != cudaSuccess) return cuda_fail(e, "advance copy");
  }
  e = record(ev3, s);
  if (e != cudaSuccess) return cuda_fail(e, "event record");
  prof_step_done(ev3, 3);
  if (queue)
    for (int i = 0; i < queue->count; ++i) queue->evals[i] += 1;
  if (pop) {
    cache->len[wslot] = n_exit;
    cache->n_advances += 1;
    if (queue) apply_pop(queue);
  }
  if (push_noise) apply_push(queue, push_rows);
  return DP_OK;
}


// ------------------------------------------------------------------ B: DiT attention sublayer

namespace {

// GEMM operand checks shared by the linear entry points: a [m][k] bf16, w [n][k] bf16.
dp_status check_linear(const void* a, const void* w, const float* bias, int64_t m, int64_t n, int64_t k) {
  if (!a || !w) return fail(DP_ERR_INVALID_ARG, "a/w NULL");
  if (!aligned16(a) || !aligned16(w) || (bias && !aligned16(bias)))
    return fail(DP_ERR_INVALID_ARG, "a/w/bias not 16-byte aligned");
  if (m <= 0 || m > INT32_MAX) return fail(DP_ERR_INVALID_ARG, "m %lld", static_cast<long long>(m));
  if (n <= 0 || n % 128 || n > INT32_MAX)
    return fail(DP_ERR_UNSUPPORTED, "n %lld (a positive multiple of 128)", static_cast<long long>(n));
  if (k <= 0 || k % 8 || k > INT32_MAX)
    return fail(DP_ERR_UNSUPPORTED, "k %lld (a positive multiple of 8)", static_cast<long long>(k));
  return DP_OK;
}

dp_status run_gemm(dp::GemmArgs& g, cudaStream_t s, const char* what) {
  dp_status st = status_ptr(&g.status);
  if (st != DP_OK) return st;
  cudaError_t e = dp::launch_gemm(g, s);
  if (e != cudaSuccess) return cuda_fail(e, what);
  return DP_OK;
}

dp::GemmArgs gemm_args(const void* a, const void* w, const float* bias, int64_t m, int32_t n, int32_t k, int epi) {
  dp::GemmArgs g;
  memset(&g, 0, sizeof(g));
  g.a = a;
  g.w = w;
  g.bias = bias;
  g.m = m;
  g.n = n;
  g.k = k;
  g.epi = epi;
  return g;
}

dp_status check_ln(const void* x, const void* h, int64_t n_rows, const dp_blocks* blk, float eps) {
  if (!x || !h || !aligned16(x) || !aligned16(h)) return fail(DP_ERR_INVALID_ARG, "x/h NULL or misaligned");
  if (!blk) return fail(DP_ERR_INVALID_ARG, "block table is NULL");
  if (!(eps > 0.0f) || !std::isfinite(eps)) return fail(DP_ERR_INVALID_ARG, "eps must be positive");
  if (n_rows <= 0 || n_rows > INT32_MAX) return fail(DP_ERR_INVALID_ARG, "n_rows %lld", static_cast<long long>(n_rows));
  if (blk->hidden % 256 || blk->hidden <= 0 || blk->hidden > 8192)
    return fail(DP_ERR_UNSUPPORTED, "hidden %d (a multiple of 256, at most 8192)", blk->hidden);
  return check_blocks(blk, n_rows, blk->hidden);
}

dp_status run_ln(const void* x, void* h, int64_t n_rows, const dp_blocks* blk, float eps, cudaStream_t s) {
  cudaError_t e = dp::launch_ln_modulate(x, h, n_rows, blk->hidden, eps, to_table(blk), s);
  if (e != cudaSuccess) return cuda_fail(e, "ln_modulate launch");
  return DP_OK;
}

dp_status run_qkv(const void* h, const void* w_qkv, const float* b_qkv, int64_t n_rows, int32_t hidden, void* q,
                  void* k, void* v, cudaStream_t s) {
  dp::GemmArgs g = gemm_args(h, w_qkv, b_qkv, n_rows, 3 * hidden, hidden, dp::kEpiQKV);
  g.y0 = q;
  g.y1 = k;
  g.y2 = v;
  g.ld_y = hidden;
  g.seg_cols = hidden;
  return run_gemm(g, s, "qkv projection launch");
}

dp_status run_out(const void* o, const void* w_o, const float* b_o, int64_t n_rows, const dp_blocks* blk,
                  const void* residual, void* out, cudaStream_t s) {
  dp::GemmArgs g = gemm_args(o, w_o, b_o, n_rows, blk->hidden, blk->hidden, dp::kEpiGateResidual);
  g.y0 = out;
  g.ld_y = blk->hidden;
  g.residual = residual;
  g.bt = to_table(blk);
  return run_gemm(g, s, "out projection launch");
}

}  // namespace

dp_status dp_ln_modulate(const void* x, void* h, int64_t n_rows, const dp_blocks* blk, float eps, void* stream) {
  dp_status st = check_ln(x, h, n_rows, blk, eps);
  if (st != DP_OK) return st;
  return run_ln(x, h, n_rows, blk, eps, static_cast<cudaStream_t>(stream));
}

dp_status dp_linear(const void* a, const void* w, const float* bias, int64_t m, int32_t n, int32_t k, void* y,
                    dp_dtype y_dt, void* stream) {
  dp_status st = check_linear(a, w, bias, m, n, k);
  if (st != DP_OK) return st;
  if (!y || !aligned16(y)) return fail(DP_ERR_INVALID_ARG, "y NULL or misaligned");
  if (y_dt != DP_BF16 && y_dt != DP_F16) return fail(DP_ERR_UNSUPPORTED, "y dtype %d (bf16 or f16)", y_dt);
  if (y == a || y == w) return fail(DP_ERR_INVALID_ARG, "y aliases an input");
  dp::GemmArgs g = gemm_args(a, w, bias, m, n, k, dp::kEpiStore);
  g.y0 = y;
  g.ld_y = n;
  g.y_f16 = y_dt == DP_F16 ? 1 : 0;
  return run_gemm(g, static_cast<cudaStream_t>(stream), "linear launch");
}

dp_status dp_qkv_project(const void* h, const void* w_qkv, const float* b_qkv, int64_t n_rows, int32_t hidden,
                         void* q, void* k, void* v, void* stream) {
  if (hidden <= 0 || hidden % 128) return fail(DP_ERR_UNSUPPORTED, "hidden %d (a multiple of 128)", hidden);
  dp_status st = check_linear(h, w_qkv, b_qkv, n_rows, 3 * static_cast<int64_t>(hidden), hidden);
  if (st != DP_OK) return st;
  if (!q || !k || !v || !aligned16(q) || !aligned16(k) || !aligned16(v))
    return fail(DP_ERR_INVALID_ARG, "q/k/v NULL or misaligned");
  if (q == h || k == h || v == h) return fail(DP_ERR_INVALID_ARG, "q/k/v alias h");
  return run_qkv(h, w_qkv, b_qkv, n_rows, hidden, q, k, v, static_cast<cudaStream_t>(stream));
}

dp_status dp_out_project(const void* o, const void* w_o, const float* b_o, int64_t n_rows, const dp_blocks* blk,
                         const void* residual, void* out, void* stream) {
  if (!blk) return fail(DP_ERR_INVALID_ARG, "block table is NULL");
  const int32_t hidden = blk->hidden;
  dp_status st = check_linear(o, w_o, b_o, n_rows, hidden, hidden);
  if (st != DP_OK) return st;
  st = check_blocks(blk, n_rows, hidden);
  if (st != DP_OK) return st;
  if (!residual || !out || !aligned16(residual) || !aligned16(out))
    return fail(DP_ERR_INVALID_ARG, "residual/out NULL or misaligned");
  if (out == o || out == w_o || out == residual) return fail(DP_ERR_INVALID_ARG, "out aliases an input");
  return run_out(o, w_o, b_o, n_rows, blk, residual, out, static_cast<cudaStream_t>(stream));
}

namespace {

// Checks shared by the fresh-context entry points: the context fits the slot the next
// attention reads, and the block table covers the context rows.  Returns that slot's k/v
// row pointers.
dp_status check_context(const dp_kvcache* cache, int64_t n_ctx, const dp_blocks* ctx_blk, dp_dtype feat,
                        char** ck, char** cv) {
  if (!ctx_blk) return fail(DP_ERR_INVALID_ARG, "context block table is NULL");
  dp_status st = check_cache(cache, ctx_blk->hidden, feat);
  if (st != DP_OK) return st;
  if (n_ctx < 0 || n_ctx > INT32_MAX) return fail(DP_ERR_INVALID_ARG, "n_ctx %lld", static_cast<long long>(n_ctx));
  if (n_ctx > cache->capacity)
    return fail(DP_ERR_CAPACITY, "context of %lld rows > cache capacity %lld", static_cast<long long>(n_ctx),
                static_cast<long long>(cache->capacity));
  st = check_blocks(ctx_blk, n_ctx, ctx_blk->hidden);
  if (st != DP_OK) return st;
  const int64_t slot_bytes = cache->capacity * ctx_blk->hidden * elem_bytes(feat);
  const int64_t slot = cache_read_slot(cache);
  *ck = static_cast<char*>(cache->k) + slot * slot_bytes;
  *cv = static_cast<char*>(cache->v) + slot * slot_bytes;
  return DP_OK;
}

// True when [a, a + na) and [b, b + nb) share a byte.
bool overlaps(const void* a, int64_t na, const void* b, int64_t nb) {
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + static_cast<uintptr_t>(nb) && y < x + static_cast<uintptr_t>(na);
}

}  // namespace

dp_status dp_context_refresh(const void* k_ctx, const void* v_ctx, int64_t n_ctx, const dp_blocks* ctx_blk,
                             dp_kvcache* cache, dp_dtype dt, void* stream) {
  if (dt != DP_BF16 && dt != DP_F32) return fail(DP_ERR_UNSUPPORTED, "context dtype %d (bf16 or f32)", dt);
  const dp_dtype feat = feature_dtype(dt);
  char* ck = nullptr;
  char* cv = nullptr;
  dp_status st = check_context(cache, n_ctx, ctx_blk, feat, &ck, &cv);
  if (st != DP_OK) return st;
  const int32_t hidden = ctx_blk->hidden;
  if (!hidden_ok(hidden, dt)) return fail(DP_ERR_INVALID_ARG, "hidden %d not a whole number of 16-byte vectors", hidden);
  if (!k_ctx || !v_ctx || !aligned16(k_ctx) || !aligned16(v_ctx))
    return fail(DP_ERR_INVALID_ARG, "k_ctx/v_ctx NULL or misaligned");
  const int64_t in_bytes = n_ctx * hidden * elem_bytes(dt);
  const int64_t ring_bytes = cache->n_slots * cache->capacity * hidden * elem_bytes(feat);
  if (overlaps(k_ctx, in_bytes, cache->k, ring_bytes) || overlaps(k_ctx, in_bytes, cache->v, ring_bytes) ||
      overlaps(v_ctx, in_bytes, cache->k, ring_bytes) || overlaps(v_ctx, in_bytes, cache->v, ring_bytes))
    return fail(DP_ERR_INVALID_ARG, "context rows overlap the cache ring");
  if (n_ctx > 0) {
    const void* src[2] = {k_ctx, v_ctx};
    void* dst[2] = {ck, cv};
    cudaError_t e = dp::launch_modulate(src, dst, 2, n_ctx, hidden, to_table(ctx_blk), dt, feat,
                                        static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "context modulate launch");
  }
  cache->len[cache_read_slot(cache)] = n_ctx;
  return DP_OK;
}

dp_status dp_context_refresh_sublayer(const void* x_ctx, int64_t n_ctx, const dp_blocks* ctx_blk, const void* w_qkv,
                                      const float* b_qkv, float eps, dp_kvcache* cache, void* work, void* stream) {
  char* ck = nullptr;
  char* cv = nullptr;
  dp_status st = check_context(cache, n_ctx, ctx_blk, DP_F16, &ck, &cv);
  if (st != DP_OK) return st;
  const int32_t hidden = ctx_blk->hidden;
  if (n_ctx > 0) {
    st = check_ln(x_ctx, work, n_ctx, ctx_blk, eps);
    if (st != DP_OK) return st;
    st = check_linear(work, w_qkv, b_qkv, n_ctx, 3 * static_cast<int64_t>(hidden), hidden);
    if (st != DP_OK) return st;
    const int64_t plane = n_ctx * hidden * 2;
    const int64_t ring_bytes = cache->n_slots * cache->capacity * hidden * 2;
    if (overlaps(work, plane, x_ctx, plane) || overlaps(work, plane, cache->k, ring_bytes) ||
        overlaps(work, plane, cache->v, ring_bytes) || overlaps(x_ctx, plane, cache->k, ring_bytes) ||
        overlaps(x_ctx, plane, cache->v, ring_bytes))
      return fail(DP_ERR_INVALID_ARG, "x_ctx, work and the cache ring must not overlap");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // B1 on the context rows, then the k and v thirds of the q/k/v projection
    st = run_ln(x_ctx, work, n_ctx, ctx_blk, eps, s);
    if (st != DP_OK) return st;
    const int64_t w_off = static_cast<int64_t>(hidden) * hidden * 2;
    dp::GemmArgs g = gemm_args(work, static_cast<const char*>(w_qkv) + w_off, b_qkv ? b_qkv + hidden : nullptr,
                               n_ctx, 2 * hidden, hidden, dp::kEpiKV);
    g.y1 = ck;
    g.y2 = cv;
    g.ld_y = hidden;
    g.seg_cols = hidden;
    st = run_gemm(g, s, "context k/v projection launch");
    if (st != DP_OK) return st;
  }
  cache->len[cache_read_slot(cache)] = n_ctx;
  return DP_OK;
}

dp_status dp_sublayer_step(const void* x, int64_t n_win, const dp_blocks* blk, const void* w_qkv, const float* b_qkv,
                           const void* w_o, const float* b_o, float eps, dp_kvcache* cache, void* work, void* out,
                           int32_t n_heads, int32_t head_dim, uint32_t flags, dp_queue* queue,
                           const void* push_noise, int64_t push_rows, void* stream) {
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (!cache) return fail(DP_ERR_INVALID_ARG, "cache is NULL");
  const int64_t hidden64 = static_cast<int64_t>(n_heads) * head_dim;
  if (n_heads <= 0 || head_dim <= 0 || hidden64 > INT32_MAX) return fail(DP_ERR_INVALID_ARG, "n_heads/head_dim");
  const int32_t hidden = static_cast<int32_t>(hidden64);
  dp_status st = check_ln(x, work, n_win, blk, eps);
  if (st != DP_OK) return st;
  if (blk->hidden != hidden) return fail(DP_ERR_INVALID_ARG, "block table hidden %d != %d", blk->hidden, hidden);
  st = check_linear(x, w_qkv, b_qkv, n_win, 3 * hidden64, hidden);
  if (st != DP_OK) return st;
  st = check_linear(x, w_o, b_o, n_win, hidden, hidden);
  if (st != DP_OK) return st;
  st = check_cache(cache, hidden, DP_F16);
  if (st != DP_OK) return st;
  if (!out || !aligned16(out)) return fail(DP_ERR_INVALID_ARG, "out NULL or misaligned");
  // work: h (bf16; later the attention output o) | q (bf16) | k (f16) | v (f16), n_win * hidden each
  const int64_t plane = n_win * hidden64 * 2;
  char* hw = static_cast<char*>(work);
  char* qw = hw + plane;
  char* kw = qw + plane;
  char* vw = kw + plane;
  if (out == work || out == x) return fail(DP_ERR_INVALID_ARG, "out aliases x or work");
  const int64_t row_bytes = hidden64 * 2;
  int64_t cache_len = 0;
  const dp::CacheSegs cseg = ring_segments(cache, flags, &cache_len);
  const char* ck = static_cast<const char*>(cache->k);
  const char* cv = static_cast<const char*>(cache->v);
  const int64_t cache_rows = static_cast<int64_t>(cache->n_slots) * cache->capacity;
  st = check_attention(qw, kw, vw, n_win, ck, cv, cache_len, nullptr, hw, n_heads, head_dim, blk, DP_BF16, DP_F16);
  if (st != DP_OK) return st;
  const bool pop = (flags & DP_STEP_POP) != 0;
  const int64_t n_exit = blk->row_offset[1];
  if (pop && n_exit > cache->capacity)
    return fail(DP_ERR_CAPACITY, "head block of %lld rows > cache capacity", static_cast<long long>(n_exit));
  if (queue) {
    st = check_queue(queue, hidden, DP_BF16);
    if (st != DP_OK) return st;
    if (pop && queue->count == 0) return fail(DP_ERR_EMPTY, "pop from an empty queue");
  }
  if (push_noise) {
    if (!queue) return fail(DP_ERR_INVALID_ARG, "push needs a queue");
    st = check_push(queue, queue->count - (pop ? 1 : 0), push_noise, push_rows);
    if (st != DP_OK) return st;
  }

  cudaEvent_t ev[kProfEvents];
  for (int i = 0; i < kProfEvents; ++i) ev[i] = prof_event(i);
  cudaError_t e = record(ev[0], s);
  if (e != cudaSuccess) return cuda_fail(e, "event record");
  // B1: h = LN(x) * (1 + scale_b) + shift_b
  st = run_ln(x, hw, n_win, blk, eps, s);
  if (st != DP_OK) return st;
  if ((e = record(ev[1], s)) != cudaSuccess) return cuda_fail(e, "event record");
  // B2: q | k | v = h W_qkv^T + b_qkv
  st = run_qkv(hw, w_qkv, b_qkv, n_win, hidden, qw, kw, vw, s);
  if (st != DP_OK) return st;
  if ((e = record(ev[2], s)) != cudaSuccess) return cuda_fail(e, "event record");
  // A2: o = attention over [cache ; window] (the modulation already happened before the projection)
  st = run_attention(qw, kw, vw, n_win, ck, cv, cseg, cache_rows, nullptr, hw, n_heads, head_dim, 0.0f, blk, 0u, DP_BF16,
                     DP_F16, s);
  if (st != DP_OK) return st;
  if ((e = record(ev[3], s)) != cudaSuccess) return cuda_fail(e, "event record");
  // B3: out = x + gate_b * (o W_o^T + b_o)
  st = run_out(hw, w_o, b_o, n_win, blk, x, out, s);
  if (st != DP_OK) return st;
  if ((e = record(ev[4], s)) != cudaSuccess) return cuda_fail(e, "event record");
  // A3: the head block's k, v -> cache ring; noise -> latent ring
  dp::CopySeg segs[dp::kMaxCopySegs];
  int nseg = 0;
  const int64_t wslot = cache->n_advances % cache->n_slots;
  if (pop) {
    segs[nseg++] = {kw, static_cast<char*>(cache->k) + wslot * cache->capacity * row_bytes, n_exit * row_bytes};
    segs[nseg++] = {vw, static_cast<char*>(cache->v) + wslot * cache->capacity * row_bytes, n_exit * row_bytes};
  }
  if (push_noise) {
    const int32_t head_after = (queue->head + (pop ? 1 : 0)) % queue->n_slots;
    const int32_t count_after = queue->count - (pop ? 1 : 0);
    const int32_t p = (head_after + count_after) % queue->n_slots;
    const int64_t bytes = push_rows * row_bytes;
    segs[nseg++] = {push_noise, queue_slot(queue, p), bytes};
    segs[nseg++] = {push_noise, queue_slot(queue, p + queue->n_slots), bytes};
  }
  if (nseg) {
    e = dp::launch_copy(segs, nseg, s);
    if (e != cudaSuccess) return cuda_fail(e, "advance copy");
  }
  if ((e = record(ev[5], s)) != cudaSuccess) return cuda_fail(e, "event record");
  prof_step_done(ev[5], 5);
  if (queue)
    for (int i = 0; i < queue->count; ++i) queue->evals[i] += 1;
  if (pop) {
    cache->len[wslot] = n_exit;
    cache->n_advances += 1;
    if (queue) apply_pop(queue);
  }
  if (push_noise) apply_push(queue, push_rows);
  return DP_OK;
}

// ------------------------------------------------------------------ the queue's schedule (host)

namespace {

// floor(b * T / W): the entry step of block b.  The pages show blocks entering one after
// another without giving the stagger; this one keeps W blocks live in the steady state and
// gives every block T evaluations.
int64_t entry_step(int64_t b, int32_t T, int32_t W) { return b * T / W; }

dp_status check_fifo(const dp_fifo* f) {
  if (!f) return fail(DP_ERR_INVALID_ARG, "schedule is NULL");
  if (f->n_blocks < 1 || f->window_blocks < 1 || f->window_blocks > DP_MAX_SLOTS ||
      f->n_timesteps < f->window_blocks)
    return fail(DP_ERR_INVALID_ARG, "schedule: n_blocks %d, T %d, W %d (need n_blocks >= 1, T >= W, 1 <= W <= %d)",
                f->n_blocks, f->n_timesteps, f->window_blocks, DP_MAX_SLOTS);
  if (f->next_block < 0 || f->next_block > f->n_blocks || f->step < 0 || f->exited_rows < 0)
    return fail(DP_ERR_INVALID_ARG, "schedule state: next_block %d, step %lld", f->next_block,
                static_cast<long long>(f->step));
  return DP_OK;
}

}  // namespace

dp_status dp_fifo_entry_step(int32_t b, int32_t n_timesteps, int32_t window_blocks, int64_t* step) {
  if (!step || b < 0 || window_blocks < 1 || n_timesteps < window_blocks)
    return fail(DP_ERR_INVALID_ARG, "entry step of block %d with T %d, W %d", b, n_timesteps, window_blocks);
  *step = entry_step(b, n_timesteps, window_blocks);
  return DP_OK;
}

dp_status dp_fifo_init(dp_fifo* f, int32_t n_blocks, int32_t n_timesteps, int32_t window_blocks) {
  if (!f) return fail(DP_ERR_INVALID_ARG, "schedule is NULL");
  dp_fifo g;
  g.n_blocks = n_blocks;
  g.n_timesteps = n_timesteps;
  g.window_blocks = window_blocks;
  g.next_block = 0;
  g.step = 0;
  g.exited_rows = 0;
  dp_status st = check_fifo(&g);
  if (st != DP_OK) return st;
  *f = g;
  return DP_OK;
}

dp_status dp_fifo_plan(const dp_fifo* f, const dp_queue* q, dp_fifo_step* out) {
  dp_status st = check_fifo(f);
  if (st != DP_OK) return st;
  if (!q || !out) return fail(DP_ERR_INVALID_ARG, "NULL argument");
  st = check_queue(q, q->hidden, q->dtype);
  if (st != DP_OK) return st;
  const int32_t T = f->n_timesteps, W = f->window_blocks;
  const int64_t s = f->step;
  dp_fifo_step o;
  o.push_before = -1;
  o.pop = 0;
  o.push_after = -1;
  o.done = 0;
  o.exit_rows = 0;
  o.ctx_rows = nullptr;
  o.ctx_n = 0;
  const int64_t total = entry_step(f->n_blocks - 1, T, W) + T;  // steps of the whole run
  if (s >= total) {
    if (q->count != 0 || f->next_block != f->n_blocks)
      return fail(DP_ERR_INVALID_ARG, "schedule finished but the queue holds %d blocks", q->count);
    o.done = 1;
    *out = o;
    return DP_OK;
  }
  if (f->next_block == 0) {
    // block 0 enters before step 0: the caller pushes it, commits, and plans again
    if (s != 0 || q->count != 0) return fail(DP_ERR_INVALID_ARG, "no block entered but step %lld, queue %d",
                                             static_cast<long long>(s), q->count);
    o.push_before = 0;
    *out = o;
    return DP_OK;
  }
  // live blocks at step s: [lo, hi), e_b <= s < e_b + T.  floor(b T / W) >= x holds exactly
  // for b >= ceil(x W / T) (x > 0), so lo and hi are the first blocks with e_b >= s - T + 1
  // and with e_b >= s + 1.
  auto first_entering_at_or_after = [&](int64_t x) -> int64_t {
    const int64_t b = x <= 0 ? 0 : (x * W + T - 1) / T;
    return b < f->n_blocks ? b : f->n_blocks;
  };
  const int64_t lo = first_entering_at_or_after(s - T + 1);
  const int64_t hi = first_entering_at_or_after(s + 1);
  if (hi != f->next_block || q->count != hi - lo)
    return fail(DP_ERR_INVALID_ARG, "queue does not match the schedule at step %lld: %d live blocks, %lld expected "
                "(blocks %lld..%lld entered, next %d)", static_cast<long long>(s), q->count,
                static_cast<long long>(hi - lo), static_cast<long long>(lo), static_cast<long long>(hi - 1),
                f->next_block);
  if (q->count < 1 || q->evals[0] != s - entry_step(lo, T, W))
    return fail(DP_ERR_INVALID_ARG, "head block has %d evaluations at step %lld, %lld expected", q->evals[0],
                static_cast<long long>(s), static_cast<long long>(s - entry_step(lo, T, W)));
  o.pop = (s - entry_step(lo, T, W) == T - 1) ? 1 : 0;
  o.exit_rows = o.pop ? q->rows[0] : 0;
  if (f->next_block < f->n_blocks && entry_step(f->next_block, T, W) == s + 1) o.push_after = f->next_block;
  // the block that left last keeps its rows in the slot behind the head until a push reuses
  // it, which cannot happen while the queue has more slots than live blocks
  if (f->exited_rows > 0 && q->n_slots > W) {
    o.ctx_rows = queue_slot(q, (q->head + q->n_slots - 1) % q->n_slots);
    o.ctx_n = f->exited_rows;
  }
  *out = o;
  return DP_OK;
}

dp_status dp_fifo_commit(dp_fifo* f, const dp_fifo_step* s) {
  dp_status st = check_fifo(f);
  if (st != DP_OK) return st;
  if (!s) return fail(DP_ERR_INVALID_ARG, "step is NULL");
  if (s->done) return fail(DP_ERR_INVALID_ARG, "the schedule is finished");
  if (s->push_before >= 0) {
    if (s->push_before != 0 || f->next_block != 0 || f->step != 0)
      return fail(DP_ERR_INVALID_ARG, "push_before %d is not the schedule's first push", s->push_before);
    f->next_block = 1;
    return DP_OK;
  }
  if (f->next_block == 0) return fail(DP_ERR_INVALID_ARG, "block 0 has not entered");
  if (s->push_after >= 0 &&
      (s->push_after != f->next_block || f->next_block >= f->n_blocks ||
       entry_step(f->next_block, f->n_timesteps, f->window_blocks) != f->step + 1))
    return fail(DP_ERR_INVALID_ARG, "push_after %d is not the block entering after step %lld", s->push_after,
                static_cast<long long>(f->step));
  if (s->push_after < 0 && f->next_block < f->n_blocks &&
      entry_step(f->next_block, f->n_timesteps, f->window_blocks) == f->step + 1)
    return fail(DP_ERR_INVALID_ARG, "block %d enters after step %lld but the plan pushes none", f->next_block,
                static_cast<long long>(f->step));
  if (s->pop && s->exit_rows <= 0) return fail(DP_ERR_INVALID_ARG, "pop of an empty block");
  f->step += 1;
  if (s->push_after >= 0) f->next_block += 1;
  if (s->pop) f->exited_rows = s->exit_rows;
  return DP_OK;
}

// ------------------------------------------------------------------ coordinated noise initialisation

dp_status dp_coordinated_frames(const int32_t* block_frames, int32_t n_blocks, int32_t window_blocks, int32_t b,
                                const int32_t* prev_frames, int32_t n_prev, const int32_t* perm,
                                int32_t* frames_out) {
  if (!block_frames || !frames_out || n_blocks < 1 || window_blocks < 1 || b < 0 || b >= n_blocks || n_prev < 0 ||
      (n_prev > 0 && !prev_frames))
    return fail(DP_ERR_INVALID_ARG, "coordinated frames: block %d of %d, W %d, %d previous frames", b, n_blocks,
                window_blocks, n_prev);
  const int32_t W = window_blocks < n_blocks ? window_blocks : n_blocks;
  int64_t pool = 0, first = 0;
  for (int32_t i = 0; i < W; ++i) {
    if (block_frames[i] < 1) return fail(DP_ERR_INVALID_ARG, "block %d has %d frames", i, block_frames[i]);
    if (i < b) first += block_frames[i];
    pool += block_frames[i];
  }
  if (pool > (1 << 24)) return fail(DP_ERR_INVALID_ARG, "pool of %lld frames", static_cast<long long>(pool));
  const int32_t nf = block_frames[b];
  if (nf < 1) return fail(DP_ERR_INVALID_ARG, "block %d has %d frames", b, nf);
  if (b < W) {
    // the first window is the pool itself, in order
    for (int32_t i = 0; i < nf; ++i) frames_out[i] = static_cast<int32_t>(first + i);
    return DP_OK;
  }
  if (!perm) return fail(DP_ERR_INVALID_ARG, "perm is NULL");
  // perm must hold every pool frame once; prev_frames are excluded
  std::vector<uint8_t> seen(static_cast<size_t>(pool), 0), excluded(static_cast<size_t>(pool), 0);
  for (int64_t i = 0; i < pool; ++i) {
    const int32_t f = perm[i];
    if (f < 0 || f >= pool || seen[f]) return fail(DP_ERR_INVALID_ARG, "perm is not a permutation of the pool");
    seen[f] = 1;
  }
  for (int32_t i = 0; i < n_prev; ++i)
    if (prev_frames[i] >= 0 && prev_frames[i] < pool) excluded[prev_frames[i]] = 1;
  int32_t got = 0;
  for (int64_t i = 0; i < pool && got < nf; ++i)
    if (!excluded[perm[i]]) frames_out[got++] = perm[i];
  if (got < nf)
    return fail(DP_ERR_INVALID_ARG, "the pool has %d frames outside the previous block, %d needed", got, nf);
  return DP_OK;
}

}  // extern "C"
