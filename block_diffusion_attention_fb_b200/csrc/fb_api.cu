// C ABI of the block-diffusion attention library (declared in include/fb.h):
// argument validation, split-KV planning, TMA descriptor creation and kernel
// launches. Every step of the path runs in the kernels of attn.cuh,
// attn_tc2.cuh, block_attn.cuh, commit.cuh, losa.cuh and cosine.cuh; this file
// only decides what to launch.
#include <cudaTypedefs.h>

#include <atomic>
#include <cmath>
#include <mutex>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <string>
#include <utility>
#include <vector>

#include "../../include/fb.h"
#include "attn.cuh"
#include "attn_tc2.cuh"
#include "block_attn.cuh"
#include "commit.cuh"
#include "cosine.cuh"
#include "losa.cuh"

// Scratch of fb_prefix_attn_noalloc: a fixed device array that every GPU which
// loads this library keeps for the life of the process. Host code may not use
// this name as a pointer (it is a host-side stand-in); the device address comes
// from cudaGetSymbolAddress, once per device.
static __device__ __align__(256) unsigned char g_fb_noalloc_scratch[FB_NOALLOC_SCRATCH_BYTES];

namespace {

using namespace fb;

thread_local std::string g_last_error;
std::atomic<unsigned long long> g_launches{0};  // kernels launched by this library

int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return code;
}

thread_local cudaError_t t_launch_error = cudaSuccess;  // of the last launch_pdl

int check_launch(const char* what) {
  cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess) e = t_launch_error;
  t_launch_error = cudaSuccess;
  if (e != cudaSuccess) return fail(FB_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return FB_OK;
}

// Launch as a programmatic dependent of the previous kernel on the stream: the
// grid may be scheduled while its predecessor finishes (every kernel of this
// library waits for its predecessor's results with griddepcontrol.wait before
// touching memory, and lets its own dependents launch right after). Inside a
// CUDA graph the edge stays programmatic. The error, if any, is reported by
// the next check_launch.
template <typename... KArgs, typename... Args>
void launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                cudaStream_t stream, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, args...);
  if (e != cudaSuccess) t_launch_error = e;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool pow2(int x) { return x > 0 && (x & (x - 1)) == 0; }
int ceil_div(long long a, long long b) { return (int)((a + b - 1) / b); }
size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
int next_pow2(int x) {
  int p = 1;
  while (p < x) p <<= 1;
  return p;
}

int sm_count() {
  static int cached[256] = {};
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 256) return 0;
  if (cached[dev]) return cached[dev];
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  cached[dev] = n;
  return n;
}

// The dynamic shared-memory limit is a per-device function attribute: raise it
// for each (device, kernel) pair when a launch needs more than was set so far.
int set_smem_once(const void* fn, int bytes) {
  struct Entry {
    int dev;
    const void* fn;
    int bytes;  // dynamic bytes the kernel may take on this device
  };
  static std::mutex mu;
  static std::vector<Entry> done;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return fail(FB_ERR_CUDA, "cudaGetDevice failed");
  std::lock_guard<std::mutex> lock(mu);
  Entry* hit = nullptr;
  for (auto& d : done)
    if (d.dev == dev && d.fn == fn) hit = &d;
  if (hit && hit->bytes >= bytes) return FB_OK;
  // the 48 KB default covers static plus dynamic shared memory
  cudaFuncAttributes fa{};
  if (cudaFuncGetAttributes(&fa, fn) != cudaSuccess)
    return fail(FB_ERR_CUDA, "cudaFuncGetAttributes failed");
  const int deflt = 48 * 1024 - (int)fa.sharedSizeBytes;
  if (bytes > deflt) {
    const cudaError_t e =
        cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess)
      return fail(FB_ERR_CUDA, "cudaFuncSetAttribute(%d bytes): %s", bytes, cudaGetErrorString(e));
  }
  const int allowed = bytes > deflt ? bytes : deflt;
  if (hit)
    hit->bytes = allowed;
  else
    done.push_back(Entry{dev, fn, allowed});
  return FB_OK;
}

size_t elem_size(fb_dtype t) { return t == FB_BF16 ? 2 : 4; }

// Tuning overrides read from the environment (0 or unset: automatic):
//   FB_SPLIT_WAVES  resident-CTA waves of the streaming (mma.sync / fp32) plan
//   FB_TC_SPLITS    splits per row tile of the tcgen05 plan
//   FB_LIST_WAVES   resident-CTA waves of page-list plans (LoSA gather, sparse residual)
int env_int(const char* name, int lo, int hi) {
  const char* e = getenv(name);
  if (e && *e) {
    const int v = atoi(e);
    if (v >= lo && v <= hi) return v;
  }
  return 0;
}

// --------------------------------------------------------------------------
// Split-KV plan: row tiles per (b, hk), and how many kTK-key tiles each CTA
// streams.
//  - Streaming kernels (HBM-bound, two CTAs per SM): one wave of CTAs. The
//    split count is the largest whose grid fits the resident slots, so every
//    CTA starts at once, streams a long key range and pays its start-up and
//    epilogue once (measured on the dllm prefix: 96 us at one wave, 110 us at
//    two, 137 us at four).
//  - tcgen05 kernel (compute-bound, one CTA per SM, long per-CTA work): the
//    split count minimises the wave-quantised makespan ceil(u*s/slots)/s plus
//    a small per-split cost (partials written and combined, per-CTA start-up);
//    caches of several sequences (lengths vary, the plan sees only the
//    longest) keep at most 128 tiles per CTA so short sequences free their
//    SMs early.
// --------------------------------------------------------------------------
struct Plan {
  int row_tile, n_row_tiles, rg;
  int tiles_per_split, n_splits;
};

// Kernel choice for bf16, head_dim 128: the tcgen05 kernel when a kv head has
// more than 64 stacked query rows (GQA groups, video blocks: its two 128-row
// Q tiles are mostly full), the mma.sync kernel for up to 64 rows (dLLM
// blocks: a 128-row MMA tile would be mostly padding while the stream is
// HBM-bound). fp32 runs on the CUDA-core kernel.
bool use_tc(fb_dtype dt, int D, int R) { return dt == FB_BF16 && D == 128 && R > 64; }

int tc_splits(long long units, int slots, int max_tiles, int batch) {
  if (const int forced = env_int("FB_TC_SPLITS", 1, 4096)) return forced;
  // cost in key-tile times: waves x (tiles per CTA + start-up) + combine reads
  int best = 1;
  double best_cost = 1e300;
  const int s_max = max_tiles < 4 * slots ? max_tiles : 4 * slots;
  for (int s = 1; s <= s_max; ++s) {
    const long long waves = (units * s + slots - 1) / slots;
    const double cost = (double)waves * (ceil_div(max_tiles, s) + 3) + 0.04 * (double)(units * s);
    if (cost < best_cost - 1e-9) {
      best_cost = cost;
      best = s;
    }
  }
  const int s_len = ceil_div(max_tiles, 128);
  if (batch > 1 && best < s_len) best = s_len;
  return best;
}

Plan make_plan(fb_dtype dt, int batch, int Hkv, int R, int max_tiles, int num_sms, int D = 128,
               bool page_list = false) {
  Plan p{};
  const int sms = num_sms > 0 ? num_sms : 148;
  max_tiles = max_tiles < 1 ? 1 : max_tiles;
  long long splits;
  if (use_tc(dt, D, R)) {
    // two 128-row Q tiles per CTA; key ranges in whole 128-key tiles (an even
    // number of 64-key metadata tiles)
    p.row_tile = kT2Rows;
    p.rg = 0;
    p.n_row_tiles = ceil_div(R, p.row_tile);
    const int tiles128 = ceil_div(max_tiles, 2);
    const int s = tc_splits((long long)batch * Hkv * p.n_row_tiles, sms, tiles128, batch);
    p.tiles_per_split = 2 * ceil_div(tiles128, s);
    p.n_splits = ceil_div(max_tiles, p.tiles_per_split);
    return p;
  } else {
    if (dt == FB_F32) {
      p.row_tile = kF32Rows;
      p.rg = 1;
    } else {
      p.rg = R <= 16 ? 1 : (R <= 32 ? 2 : 4);
      p.row_tile = 16 * p.rg;
    }
    p.n_row_tiles = ceil_div(R, p.row_tile);
    const long long units = (long long)batch * Hkv * p.n_row_tiles;
    int waves = env_int("FB_SPLIT_WAVES", 1, 64);
    if (page_list) {
      // Page lists are planned on their upper bound (the counts live on the
      // device). Several sequences have unions of different sizes, so a second
      // wave lets the CTA scheduler balance them (measured, batch-8 GQA LoSA:
      // 590 us per step at one wave, 400 at two, 409 at four; single-sequence
      // workloads are fastest at one wave).
      waves = env_int("FB_LIST_WAVES", 1, 64);
      if (!waves) waves = batch > 1 ? 2 : 1;
    }
    splits = (long long)sms * 2 * (waves ? waves : 1) / units;
  }
  if (splits < 1) splits = 1;
  if (splits > max_tiles) splits = max_tiles;
  p.tiles_per_split = ceil_div(max_tiles, splits);
  p.n_splits = ceil_div(max_tiles, p.tiles_per_split);
  return p;
}

// Split partials [splits, batch, Hkv, R, D] + their log2 normalisers.
size_t partial_bytes(const Plan& p, int batch, int Hkv, int R, int D) {
  if (p.n_splits <= 1) return 0;
  const size_t rows = (size_t)p.n_splits * batch * Hkv * R;
  return round_up(rows * D * 4, 256) + round_up(rows * 4, 256);
}

// Workspace bytes of one attention-partial launch (split partials).
// Page-list attention (LoSA gather, sparse residual) runs on the same split grid
// kernels as dense prefixes: measured against a persistent stream-K kernel it
// was faster on every page-list workload (dllm LoSA 108.6 vs 122.8 us per step,
// sparse residual 96.6 vs 159.0; L = 131072: 180.9 vs 205.2 and 245.0 vs 343.5),
// whose short per-CTA tile runs were latency-bound on group merges.
size_t partial_ws_bytes(fb_dtype dt, int batch, int Hkv, int R, int D, int max_tiles,
                        int num_sms, bool page_list = false) {
  return partial_bytes(make_plan(dt, batch, Hkv, R, max_tiles, num_sms, D, page_list), batch, Hkv,
                       R, D);
}

// Workspace regions shared by every entry point (offsets in bytes).
struct WsLayout {
  size_t part, scores, tickets, cos, a_in, l_in, total;
};

int logical_pages(const fb_kv* kv) {
  return kv->page_table ? kv->max_pages_per_seq : ceil_div(kv->max_seq_len, kv->page_size);
}

int max_union_entries(const fb_kv* kv, int G, int n_active, int topk) {
  const long long u = (long long)n_active * G * topk;
  const int np = logical_pages(kv);
  return (int)(u < np ? u : np);
}

WsLayout ws_layout(const fb_kv* kv, int B, int Hq, int n_active, int topk, int num_sms) {
  WsLayout w{};
  const int G = Hq / kv->n_heads_kv, D = kv->head_dim;
  const int R = B * G;
  size_t part = partial_ws_bytes(kv->dtype, kv->batch, kv->n_heads_kv, R, D,
                                 ceil_div(kv->max_seq_len, kTK), num_sms);
  size_t scores = 0, tickets = 0;
  if (n_active > 0 && topk > 0) {
    const int na = n_active < B ? n_active : B;
    const int per_tile = kTK / (kv->page_size < kTK ? kv->page_size : kTK);
    const int ent = max_union_entries(kv, G, na, topk);
    const size_t pgb = partial_ws_bytes(kv->dtype, kv->batch, kv->n_heads_kv, na * G, D,
                                        ceil_div(ent, per_tile), num_sms, true);
    part = part > pgb ? part : pgb;
    scores = round_up((size_t)kv->batch * na * Hq * logical_pages(kv) * 4, 256) +
             round_up((size_t)kv->batch * B * 4, 256);
    tickets = round_up((size_t)kv->batch * kv->n_heads_kv * 4, 256);  // top-k group tickets
  }
  const int P = next_pow2(B * D);
  const int T1 = P < kCosT1Max ? P : kCosT1Max;
  const size_t cosb = round_up((size_t)kv->batch * Hq * 3 * T1 * 8, 256);
  w.part = 0;
  w.scores = w.part + part;
  w.tickets = w.scores + scores;
  w.cos = w.tickets + tickets;
  w.a_in = w.cos + cosb;
  w.l_in = w.a_in + round_up((size_t)kv->batch * B * Hq * D * 4, 256);
  w.total = w.l_in + round_up((size_t)kv->batch * B * Hq * 4, 256);
  return w;
}

// --------------------------------------------------------------------------
// TMA descriptors for the K / V pools: 3-D view [n_slots][Hkv][D] bf16, boxes
// of 64 channels (128 bytes, swizzled) x 1 head x `chunk` tokens.
// --------------------------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

int make_tmap(CUtensorMap* m, const void* base, int D, int Hkv, long long n_slots, int chunk) {
  auto fn = encode_fn();
  if (!fn) return fail(FB_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)Hkv, (cuuint64_t)n_slots};
  cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)Hkv * D * 2};
  cuuint32_t box[3] = {64, 1, (cuuint32_t)chunk};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(FB_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return FB_OK;
}

// packed: a varlen block's own keys (rows of each sequence given by offsets,
// so the per-sequence capacity check of a contiguous cache does not apply)
int validate_kv(const fb_kv* kv, bool packed = false) {
  if (!kv) return fail(FB_ERR_ARG, "kv is NULL");
  if (!kv->k || !kv->v) return fail(FB_ERR_ARG, "kv->k / kv->v is NULL");
  if (kv->batch <= 0 || kv->batch > 256) return fail(FB_ERR_ARG, "batch must be in [1, 256]");
  if (kv->n_heads_kv <= 0 || kv->max_seq_len < 0 || kv->n_slots <= 0)
    return fail(FB_ERR_ARG, "bad kv sizes");
  if (kv->n_slots >= (1LL << 31)) return fail(FB_ERR_SHAPE, "n_slots must be < 2^31");
  if (kv->head_dim != 64 && kv->head_dim != 128)
    return fail(FB_ERR_SHAPE, "head_dim %d unsupported (64, 128)", kv->head_dim);
  if (kv->dtype != FB_BF16 && kv->dtype != FB_F32) return fail(FB_ERR_ARG, "bad dtype");
  if (!pow2(kv->page_size) || kv->page_size < 16)
    return fail(FB_ERR_SHAPE, "page_size must be a power of two >= 16");
  if (kv->page_table && kv->max_pages_per_seq * (long long)kv->page_size < kv->max_seq_len)
    return fail(FB_ERR_ARG, "max_pages_per_seq * page_size < max_seq_len");
  if (!packed && !kv->page_table && (long long)kv->batch * kv->max_seq_len > kv->n_slots)
    return fail(FB_ERR_ARG, "contiguous cache needs batch * max_seq_len <= n_slots");
  if (!aligned16(kv->k) || !aligned16(kv->v)) return fail(FB_ERR_ALIGN, "k / v not 16-byte aligned");
  return FB_OK;
}

// Shared launcher of the attention partial (prefix, block, or LoSA gather).
struct PartialCall {
  const void* q;
  int B, Hq;
  float scale;
  const fb_kv* kv;
  const int32_t* row_list;
  int n_list;
  const int32_t* page_list;
  const int32_t* page_count;
  int page_list_stride, max_list_entries;
  const uint8_t* head_mask;
  const unsigned long long* seq_bits;  // 4 words or NULL
  float* a_out;
  float* l_out;
  float* a_prev;
  void* ws;
  size_t ws_bytes;
  size_t ws_offset;
  int num_sms;
  bool single_split;  // one CTA streams the whole key set (no workspace)
  const float* mrg_a;  // optional: merge every final row with this partial (FlashBlock merge)
  const float* mrg_l;
  const int32_t* q_cu;   // optional: packed query rows (device [batch + 1] offsets), q_total rows
  int q_total;
  const int32_t* kv_cu;  // optional: packed contiguous key set (device [batch + 1] offsets)
};

// The kernels order keys by raw score when forming the row maximum, which
// needs a positive scale.
int validate_scale(float scale) {
  if (!(scale > 0.f) || !std::isfinite(scale))
    return fail(FB_ERR_ARG, "scale must be positive and finite (got %g)", (double)scale);
  return FB_OK;
}

int launch_partial(const PartialCall& c, cudaStream_t stream) {
  if (int rc_ = validate_scale(c.scale)) return rc_;
  {
    // One sequence whose stacked rows leave a last 256-row tile of at most 64
    // rows (a video block of 1560 rows: 6 full tiles and 24 rows): on the
    // tcgen05 kernel that tile costs as much as a full one and pushes the grid
    // into another wave (video prefix: 7 x 24 tiles x 4 splits = 4.5 waves).
    // With a workspace, the full tiles run on the tcgen05 kernel (video: 144
    // CTAs, one wave, no split) and the last rows on the streaming kernel,
    // which reads the key set once more at its HBM rate; each part writes (and
    // merges) its own rows.
    const fb_kv* kv = c.kv;
    const int G = c.Hq / kv->n_heads_kv, R = c.B * G, tail = R % kT2Rows;
    if (!c.single_split && c.ws && kv->batch == 1 && !c.q_cu && !c.row_list && !c.page_list &&
        use_tc(kv->dtype, kv->head_dim, R) && R > kT2Rows && tail > 0 && tail <= 64 &&
        tail % G == 0) {
      const int Bt = tail / G, Bm = c.B - Bt;
      const int max_tiles = ceil_div(kv->max_seq_len, kTK);
      const Plan pm = make_plan(kv->dtype, 1, kv->n_heads_kv, Bm * G, max_tiles, c.num_sms,
                                kv->head_dim);
      const Plan pt = make_plan(kv->dtype, 1, kv->n_heads_kv, tail, max_tiles, c.num_sms,
                                kv->head_dim);
      const size_t nm = partial_bytes(pm, 1, kv->n_heads_kv, Bm * G, kv->head_dim);
      const size_t nt = partial_bytes(pt, 1, kv->n_heads_kv, tail, kv->head_dim);
      const long long r0 = (long long)Bm * c.Hq;  // first (row, head) of the last rows
      const int D = kv->head_dim;
      const void* qt = static_cast<const char*>(c.q) + r0 * D * elem_size(kv->dtype);
      if (c.ws_offset + (nm > nt ? nm : nt) <= c.ws_bytes && aligned16(qt)) {
        PartialCall cm = c, ct = c;
        cm.B = Bm;
        ct.q = qt;
        ct.B = Bt;
        ct.a_out = c.a_out + r0 * D;
        ct.l_out = c.l_out + r0;
        ct.a_prev = c.a_prev ? c.a_prev + r0 * D : nullptr;
        ct.mrg_a = c.mrg_a ? c.mrg_a + r0 * D : nullptr;
        ct.mrg_l = c.mrg_l ? c.mrg_l + r0 : nullptr;
        if (int rc_ = launch_partial(cm, stream)) return rc_;
        return launch_partial(ct, stream);
      }
    }
  }
  const fb_kv* kv = c.kv;
  const int D = kv->head_dim, Hkv = kv->n_heads_kv, G = c.Hq / Hkv;
  AttnArgs a{};
  a.q = c.q;
  a.k = kv->k;
  a.v = kv->v;
  a.batch = kv->batch;
  a.B = c.B;
  a.Hq = c.Hq;
  a.Hkv = Hkv;
  a.G = G;
  a.row_list = c.row_list;
  a.n_list = c.n_list;
  a.R = (c.row_list ? c.n_list : c.B) * G;
  a.page_table = kv->page_table;
  a.max_pages = kv->max_pages_per_seq;
  a.page_size = kv->page_size;
  a.seq_len = kv->seq_len;
  a.max_seq_len = kv->max_seq_len;
  a.page_list = c.page_list;
  a.page_count = c.page_count;
  a.page_list_stride = c.page_list_stride;
  a.n_slots = kv->n_slots;
  a.head_mask = c.head_mask;
  if (c.seq_bits) {
    a.use_seq_bits = 1;
    for (int i = 0; i < 4; ++i) a.seq_bits[i] = c.seq_bits[i];
  }
  a.scale_log2 = c.scale * kLog2e;
  a.mrg_a = c.mrg_a;
  a.mrg_l = c.mrg_l;
  if (c.q_cu && c.row_list) return fail(FB_ERR_ARG, "packed rows cannot take a row list");
  a.q_cu = c.q_cu;
  a.q_total = c.q_total;
  a.kv_cu = c.kv_cu;
  a.a_out = c.a_out;
  a.l_out = c.l_out;
  a.a_prev = c.a_prev;
  if (a.R == 0) return FB_OK;
  int max_tiles;
  if (c.page_list) {
    if (kv->page_size > kTK) return fail(FB_ERR_SHAPE, "page-list attention needs page_size <= 64");
    a.chunk = kv->page_size;
    max_tiles = ceil_div(c.max_list_entries, kTK / kv->page_size);
  } else {
    a.chunk = kv->page_table ? (kv->page_size < kTK ? kv->page_size : kTK) : kTK;
    max_tiles = ceil_div(kv->max_seq_len, kTK);
  }
  Plan p = make_plan(kv->dtype, kv->batch, Hkv, a.R, max_tiles, c.num_sms, D,
                     c.page_list != nullptr);
  if (c.single_split) {
    p.tiles_per_split = max_tiles < 1 ? 1 : max_tiles;
    p.n_splits = 1;
  }
  a.row_tile = p.row_tile;
  a.n_row_tiles = p.n_row_tiles;
  a.tiles_per_split = p.tiles_per_split;
  a.n_splits = p.n_splits;
  const size_t need = partial_bytes(p, kv->batch, Hkv, a.R, D);
  if (need > 0) {
    if (!c.ws || c.ws_offset + need > c.ws_bytes)
      return fail(FB_ERR_WORKSPACE, "workspace too small: need %zu bytes at offset %zu, have %zu",
                  need, c.ws_offset, c.ws_bytes);
    if (!aligned16(c.ws)) return fail(FB_ERR_ALIGN, "workspace not 16-byte aligned");
    const size_t rows = (size_t)p.n_splits * kv->batch * Hkv * a.R;
    char* w = static_cast<char*>(c.ws) + c.ws_offset;
    a.o_part = reinterpret_cast<float*>(w);
    a.lse_part = reinterpret_cast<float*>(w + round_up(rows * D * 4, 256));
  }
  const dim3 grid(p.n_row_tiles * p.n_splits, Hkv, kv->batch);
  if (kv->dtype == FB_F32) {
#define FB_LAUNCH_F32(DD)                                                         \
  do {                                                                            \
    auto kfn = attn_f32_kernel<DD>;                                               \
    if (int rc_ = set_smem_once((const void*)kfn, F32Smem<DD>::bytes)) return rc_; \
    launch_pdl(kfn, grid, dim3(128), F32Smem<DD>::bytes, stream, a);              \
  } while (0)
    if (D == 128)
      FB_LAUNCH_F32(128);
    else
      FB_LAUNCH_F32(64);
#undef FB_LAUNCH_F32
  } else {
    CUtensorMap tk, tv;
    int rc = make_tmap(&tk, kv->k, D, Hkv, kv->n_slots, a.chunk);
    if (rc) return rc;
    rc = make_tmap(&tv, kv->v, D, Hkv, kv->n_slots, a.chunk);
    if (rc) return rc;
#define FB_LAUNCH_BF16(DD, RGV)                                                              \
  do {                                                                                       \
    auto kfn = attn_bf16_kernel<DD, RGV>;                                                    \
    const int smem = Bf16Smem<DD>::kBytes;                                                   \
    if (int rc_ = set_smem_once((const void*)kfn, smem)) return rc_;                       \
    launch_pdl(kfn, grid, dim3(kAttnThreads), smem, stream, a, tk, tv);                      \
  } while (0)
    if (use_tc(kv->dtype, D, a.R)) {
      if (int rc_ = set_smem_once((const void*)attn_tc2_kernel, Tc2Smem::kBytes)) return rc_;
      launch_pdl(attn_tc2_kernel, grid, dim3(kT2Threads), Tc2Smem::kBytes, stream, a, tk, tv);
    } else if (D == 128) {
      if (p.rg == 1)
        FB_LAUNCH_BF16(128, 1);
      else if (p.rg == 2)
        FB_LAUNCH_BF16(128, 2);
      else
        FB_LAUNCH_BF16(128, 4);
    } else {
      if (p.rg == 1)
        FB_LAUNCH_BF16(64, 1);
      else if (p.rg == 2)
        FB_LAUNCH_BF16(64, 2);
      else
        FB_LAUNCH_BF16(64, 4);
    }
#undef FB_LAUNCH_BF16
  }
  int rc = check_launch("attention partial kernel");
  if (rc) return rc;
  if (p.n_splits > 1) {
    const long long rows = (long long)kv->batch * Hkv * a.R;
    const int blocks = ceil_div(rows * 32, 256);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(blocks);
    cfg.blockDim = dim3(256);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = D == 128 ? cudaLaunchKernelEx(&cfg, combine_kernel<128>, a)
                                   : cudaLaunchKernelEx(&cfg, combine_kernel<64>, a);
    if (e != cudaSuccess)
      return fail(FB_ERR_CUDA, "split combine kernel launch: %s", cudaGetErrorString(e));
    rc = check_launch("split combine kernel");
  }
  return rc;
}

int validate_q(const void* q, int B, int Hq, const fb_kv* kv) {
  if (!q) return fail(FB_ERR_ARG, "q is NULL");
  if (B <= 0 || Hq <= 0) return fail(FB_ERR_ARG, "B and n_heads_q must be positive");
  if (Hq % kv->n_heads_kv) return fail(FB_ERR_SHAPE, "n_heads_q %% n_heads_kv != 0");
  if (!aligned16(q)) return fail(FB_ERR_ALIGN, "q not 16-byte aligned");
  return FB_OK;
}

int merge_launch(const float* ao, const float* lo, const float* ai, const float* li, long long rows,
                 int D, float* af, float* lf, cudaStream_t stream) {
  if (rows == 0) return FB_OK;
  const int blocks = ceil_div(rows * 32, 256);
  if (D == 128)
    merge_kernel<128><<<blocks, 256, 0, stream>>>(ao, lo, ai, li, rows, af, lf);
  else
    merge_kernel<64><<<blocks, 256, 0, stream>>>(ao, lo, ai, li, rows, af, lf);
  return check_launch("merge kernel");
}

KvView kv_view(const fb_kv* kv) {
  KvView v{};
  v.k = kv->k;
  v.page_table = kv->page_table;
  v.seq_len = kv->seq_len;
  v.n_slots = kv->n_slots;
  v.batch = kv->batch;
  v.Hkv = kv->n_heads_kv;
  v.D = kv->head_dim;
  v.page_size = kv->page_size;
  v.max_pages = kv->page_table ? kv->max_pages_per_seq : ceil_div(kv->max_seq_len, kv->page_size);
  v.max_seq_len = kv->max_seq_len;
  return v;
}

// Page scoring grid: chunks of kPsPages pages per (sequence, kv head), `cpc`
// consecutive chunks per CTA so that the grid is ONE wave of the CTAs an SM
// holds at this shared-memory size (up to two): a second, partial wave would
// double the time of the chunks it runs.
dim3 page_score_grid(const KvView& v, int num_sms, int smem_bytes, int& cpc) {
  const int chunks = ceil_div(v.max_pages, kPsPages);
  const long long groups = (long long)v.batch * v.Hkv;
  const int per_sm = smem_bytes + 1024 <= (227 * 1024) / 2 ? 2 : 1;
  const long long slots = (long long)per_sm * (num_sms > 0 ? num_sms : 148);
  cpc = (int)((groups * chunks + slots - 1) / slots);
  if (cpc < 1) cpc = 1;
  if (cpc > chunks) cpc = chunks;
  while (cpc < chunks && (long long)ceil_div(chunks, cpc) * groups > slots) ++cpc;
  return dim3(ceil_div(chunks, cpc), v.Hkv, v.batch);
}

// Grid of the bf16 page scorer: tiles of kPcPages pages per (sequence, kv
// head), `tpc` consecutive tiles per CTA (a multiple of its warps, which take
// them in turn), as few as keep the grid within one wave.
dim3 page_cols_grid(const KvView& v, int num_sms, int smem_bytes, int& tpc) {
  constexpr int nw = kPcThreads / 32;
  const int tiles = ceil_div(v.max_pages, kPcPages);
  const long long groups = (long long)v.batch * v.Hkv;
  const int per_sm = smem_bytes + 1024 <= (227 * 1024) / 2 ? 2 : 1;
  const long long slots = (long long)per_sm * (num_sms > 0 ? num_sms : 148);
  tpc = (int)((groups * tiles + slots - 1) / slots);
  tpc = ceil_div(tpc < 1 ? 1 : tpc, nw) * nw;
  while (tpc < tiles && (long long)ceil_div(tiles, tpc) * groups > slots) tpc += nw;
  return dim3(ceil_div(tiles, tpc), v.Hkv, v.batch);
}

// Short blocks (bf16, B <= 64): the latency-built kernel of block_attn.cuh.
// Rows per CTA: 16 per warp, 1 to 4 warps, fewer warps while that keeps the
// grid within two CTAs per SM (more CTAs = more of the block's loads in flight).
int block_attn_short(const void* q, const void* k_in, const void* v_in, int batch, int B, int Hq,
                     int Hkv, int D, float scale, float* a_out, float* l_out, const float* mrg_a,
                     const float* mrg_l, const int32_t* cu, int total, cudaStream_t stream) {
  if (int rc_ = validate_scale(scale)) return rc_;
  BlockArgs a{};
  a.cu = cu;
  a.total = total;
  a.q = static_cast<const __nv_bfloat16*>(q);
  a.k = static_cast<const __nv_bfloat16*>(k_in);
  a.v = static_cast<const __nv_bfloat16*>(v_in);
  a.mrg_a = mrg_a;
  a.mrg_l = mrg_l;
  a.a_out = a_out;
  a.l_out = l_out;
  a.batch = batch;
  a.B = B;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.G = Hq / Hkv;
  a.R = B * a.G;
  a.scale_log2 = scale * kLog2e;
  if (batch == 0 || B == 0) return FB_OK;
  if (!aligned16(mrg_a)) return fail(FB_ERR_ALIGN, "merge partner rows not 16-byte aligned");
  const int tiles16 = ceil_div(a.R, 16);
  const long long groups = (long long)batch * Hkv;
  const int slots = 2 * (sm_count() > 0 ? sm_count() : 148);
  int warps = 1;
  while (warps < 4 && warps < tiles16 && groups * ceil_div(tiles16, warps) > slots) warps *= 2;
  const int kt = ceil_div(B, 16);
  const int smem = BlockSmem<128>::bytes(warps, kt, mrg_a != nullptr);
  const int smem_d = D == 128 ? smem : BlockSmem<64>::bytes(warps, kt, mrg_a != nullptr);
  const dim3 grid(ceil_div(a.R, 16 * warps), Hkv, batch);
  if (grid.y > 65535 || grid.z > 65535) return fail(FB_ERR_SHAPE, "too many heads or sequences");
#define FB_BLOCK_LAUNCH(DD, KTV)                                                       \
  do {                                                                                 \
    auto kfn = block_attn_kernel<DD, KTV>;                                             \
    if (int rc_ = set_smem_once((const void*)kfn, smem_d)) return rc_;                \
    launch_pdl(kfn, grid, dim3(32 * warps), smem_d, stream, a);                        \
  } while (0)
  if (D == 128) {
    switch (kt) {
      case 1: FB_BLOCK_LAUNCH(128, 1); break;
      case 2: FB_BLOCK_LAUNCH(128, 2); break;
      case 3: FB_BLOCK_LAUNCH(128, 3); break;
      default: FB_BLOCK_LAUNCH(128, 4); break;
    }
  } else {
    switch (kt) {
      case 1: FB_BLOCK_LAUNCH(64, 1); break;
      case 2: FB_BLOCK_LAUNCH(64, 2); break;
      case 3: FB_BLOCK_LAUNCH(64, 3); break;
      default: FB_BLOCK_LAUNCH(64, 4); break;
    }
  }
#undef FB_BLOCK_LAUNCH
  return check_launch("block attention kernel");
}

// Short fp32 blocks (B <= 64): one CTA of up to 8 warps per (sequence, kv head).
int block_attn_short_f32(const void* q, const void* k_in, const void* v_in, int batch, int B,
                         int Hq, int Hkv, int D, float scale, float* a_out, float* l_out,
                         const float* mrg_a, const float* mrg_l, const int32_t* cu, int total,
                         cudaStream_t stream) {
  if (int rc_ = validate_scale(scale)) return rc_;
  BlockArgsF32 a{};
  a.cu = cu;
  a.total = total;
  a.q = static_cast<const float*>(q);
  a.k = static_cast<const float*>(k_in);
  a.v = static_cast<const float*>(v_in);
  a.mrg_a = mrg_a;
  a.mrg_l = mrg_l;
  a.a_out = a_out;
  a.l_out = l_out;
  a.batch = batch;
  a.B = B;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.G = Hq / Hkv;
  a.R = B * a.G;
  a.scale = scale;
  if (batch == 0 || B == 0) return FB_OK;
  if (batch > 65535) return fail(FB_ERR_SHAPE, "too many sequences");
  const int warps = a.R < 8 ? a.R : 8;
  const int smem = block_f32_smem(D, a.R);
#define FB_BLOCK_F32_LAUNCH(DD)                                          \
  do {                                                                   \
    auto kfn = block_attn_f32_kernel<DD>;                                \
    if (int rc_ = set_smem_once((const void*)kfn, smem)) return rc_;    \
    launch_pdl(kfn, dim3(Hkv, batch), dim3(32 * warps), smem, stream, a); \
  } while (0)
  if (D == 128)
    FB_BLOCK_F32_LAUNCH(128);
  else
    FB_BLOCK_F32_LAUNCH(64);
#undef FB_BLOCK_F32_LAUNCH
  return check_launch("fp32 block attention kernel");
}

// Block-internal partial of every block row (optionally merged with mrg_a /
// mrg_l). Packed rows (cu != NULL): sequence b's rows and keys are rows
// cu[b] .. cu[b+1]-1 of the total packed rows, at most B of them.
int block_attn_impl(const void* q, const void* k_in, const void* v_in, int batch, int B, int Hq,
                    int Hkv, int D, float scale, fb_dtype dt, float* a_in, float* l_in,
                    cudaStream_t stream, const float* mrg_a = nullptr,
                    const float* mrg_l = nullptr, const int32_t* cu = nullptr, int total = 0,
                    void* ws = nullptr, size_t ws_bytes = 0, size_t ws_offset = 0) {
  fb_kv kv{};
  kv.k = k_in;
  kv.v = v_in;
  kv.n_slots = cu ? (long long)(total > 0 ? total : 1) : (long long)batch * B;
  kv.batch = batch;
  kv.n_heads_kv = Hkv;
  kv.head_dim = D;
  kv.page_size = 16;
  kv.max_seq_len = B;
  kv.dtype = dt;
  int rc = validate_kv(&kv, cu != nullptr);
  if (rc) return rc;
  rc = validate_q(q, B, Hq, &kv);
  if (rc) return rc;
  if (!a_in || !l_in) return fail(FB_ERR_ARG, "a_in / l_in is NULL");
  if (mrg_a && !mrg_l) return fail(FB_ERR_ARG, "merge partner without its L");
  if (cu && total == 0) return FB_OK;  // no rows at all
  if (dt == FB_BF16 && (D == 64 || D == 128) && B <= 64) return block_attn_short(
      q, k_in, v_in, batch, B, Hq, Hkv, D, scale, a_in, l_in, mrg_a, mrg_l, cu, total, stream);
  if (dt == FB_F32 && (D == 64 || D == 128) && B <= 64 &&
      block_f32_smem(D, B * (Hq / Hkv)) <= 200 * 1024)
    return block_attn_short_f32(q, k_in, v_in, batch, B, Hq, Hkv, D, scale, a_in, l_in, mrg_a,
                                mrg_l, cu, total, stream);
  PartialCall c{};
  c.q = q;
  c.B = B;
  c.Hq = Hq;
  c.scale = scale;
  c.kv = &kv;
  c.a_out = a_in;
  c.l_out = l_in;
  // the block is short: one split per (b, hk, row tile) and no workspace,
  // unless the caller lends one (launch_partial may then split off a short
  // last row tile)
  c.single_split = ws == nullptr;
  c.ws = ws;
  c.ws_bytes = ws_bytes;
  c.ws_offset = ws_offset;

  c.num_sms = sm_count();
  c.mrg_a = mrg_a;
  c.mrg_l = mrg_l;
  c.q_cu = cu;
  c.q_total = total;
  c.kv_cu = cu;
  return launch_partial(c, stream);
}

// Selection of the sparse-residual mode: per (sequence, kv head) the top-k
// pages by head score (max over block rows and the kv head's q heads of the
// QUEST-style bound) into bitmap / list / count, the other pages of the
// sequence into comp_list / comp_count.
int sr_select(const void* q, int B, int Hq, const void* page_min, const void* page_max,
              const fb_kv* kv, int topk, uint32_t* bitmap, int32_t* list, int32_t* count,
              int32_t* comp_list, int32_t* comp_count, float* head_scores, int* tickets,
              cudaStream_t stream) {
  const KvView v = kv_view(kv);
  const int D = v.D, G = Hq / v.Hkv, RQ = B * G;
  const int words = ceil_div(v.max_pages, 32);

  if (v.max_pages > 32768) return fail(FB_ERR_SHAPE, "sparse residual supports <= 32768 pages");
  if (!aligned16(page_min) || !aligned16(page_max))
    return fail(FB_ERR_ALIGN, "page summaries not 16-byte aligned");
  int rc;
  if (kv->dtype == FB_BF16) {
    int tpc;
    const int psm = page_score_cols_smem(RQ, D, true);
    const dim3 g2 = page_cols_grid(v, sm_count(), psm, tpc);
    auto kfn = D == 128 ? page_score_cols_kernel<128, kPcHeadMax>
                        : page_score_cols_kernel<64, kPcHeadMax>;
    if ((rc = set_smem_once((const void*)kfn, psm))) return rc;
    launch_pdl(kfn, g2, dim3(kPcThreads), psm, stream, static_cast<const __nv_bfloat16*>(q),
               (const int32_t*)nullptr, (const float*)nullptr, (int32_t*)nullptr, B, Hq, G, B,
               static_cast<const __nv_bfloat16*>(page_min),
               static_cast<const __nv_bfloat16*>(page_max), v, head_scores, bitmap, words,
               tickets, tpc);
  } else {
    int cpc;
    const int psm = page_score_smem(RQ < kHsRows ? RQ : kHsRows, D);
    const dim3 g2 = page_score_grid(v, sm_count(), psm, cpc);
    auto kfn = D == 128 ? head_page_score_kernel<float, 128> : head_page_score_kernel<float, 64>;
    if ((rc = set_smem_once((const void*)kfn, psm))) return rc;
    launch_pdl(kfn, g2, dim3(256), psm, stream, static_cast<const float*>(q), B, Hq, G,
               static_cast<const float*>(page_min), static_cast<const float*>(page_max), v,
               head_scores, bitmap, words, tickets, cpc);
  }
  if ((rc = check_launch("head page score kernel"))) return rc;
  const int ksm = (v.max_pages + words) * 4;
  if ((rc = set_smem_once((const void*)topk_pages_kernel, ksm))) return rc;
  // one "row" per kv head: scores [batch, 1, Hkv, pages], G = 1; each CTA is its
  // own group and compacts its selection
  launch_pdl(topk_pages_kernel, dim3(v.Hkv, kv->batch), dim3(kTopkThreads), ksm, stream,
             (const float*)head_scores, v, v.Hkv, 1, 1, topk, bitmap, words, list, count,
             v.max_pages, tickets);
  if ((rc = check_launch("top-k pages kernel"))) return rc;
  launch_pdl(complement_compact_kernel, dim3(v.Hkv, kv->batch), dim3(256), 0, stream,
             (const uint32_t*)bitmap, words, v, v.max_pages, comp_list, comp_count);
  return check_launch("complement compaction kernel");
}

}  // namespace

extern "C" {

const char* fb_last_error(void) { return g_last_error.c_str(); }

uint64_t fb_kernel_launches(void) { return g_launches.load(std::memory_order_relaxed); }

int fb_device_status(void) {
  int word = 0, zero = 0;
  if (cudaDeviceSynchronize() != cudaSuccess) return fail(FB_ERR_CUDA, "device synchronize failed");
  if (cudaMemcpyFromSymbol(&word, g_fb_error_word, sizeof(int)) != cudaSuccess)
    return fail(FB_ERR_CUDA, "reading the device error word failed");
  cudaMemcpyToSymbol(g_fb_error_word, &zero, sizeof(int));
  if (word & kErrBadPage)
    return fail(FB_ERR_ARG, "fb_block_commit met a page-table entry outside the pool (that page "
                            "was left unwritten)");
  if (word & kErrBadReadPage)
    return fail(FB_ERR_ARG, "a page-table entry outside the pool was read (its tokens were "
                            "treated as absent)");
  if (word & kErrBadRows)
    return fail(FB_ERR_ARG, "packed row offsets left the buffer, decreased or exceeded the most "
                            "rows per sequence (that sequence was treated as empty)");
  if (word) return fail(FB_ERR_TIMEOUT, "a device-side wait exceeded its budget");
  return FB_OK;
}

int fb_selftest_timeout(int32_t* gave_up, cudaStream_t stream) {
  selftest_wait_kernel<<<1, 32, 0, stream>>>(2000000LL, gave_up);  // about a millisecond
  return check_launch("self-test wait kernel");
}

int fb_block_commit(const fb_kv* kv, const int32_t* seq_len_host, const void* k_in,
                    const void* v_in, int32_t B, void* page_min, void* page_max,
                    cudaStream_t stream) {
  int rc = validate_kv(kv);
  if (rc) return rc;
  if (!kv->seq_len) return fail(FB_ERR_ARG, "kv->seq_len is NULL: the lengths are updated in place");
  if (!seq_len_host) return fail(FB_ERR_ARG, "seq_len_host is NULL");
  if (B < 0) return fail(FB_ERR_ARG, "B must be >= 0");
  if (B > 0 && (!k_in || !v_in)) return fail(FB_ERR_ARG, "k_in / v_in is NULL");
  if ((page_min == nullptr) != (page_max == nullptr))
    return fail(FB_ERR_ARG, "page_min and page_max must both be given or both be NULL");
  if (!aligned16(k_in) || !aligned16(v_in)) return fail(FB_ERR_ALIGN, "k_in / v_in not 16-byte aligned");
  const KvView v = kv_view(kv);
  CommitArgs a{};
  int max_touched = 0;
  for (int b = 0; b < kv->batch; ++b) {
    const int n = seq_len_host[b];
    if (n < 0 || (long long)n + B > kv->max_seq_len)
      return fail(FB_ERR_ARG, "sequence %d: %d + %d tokens exceed max_seq_len %d", b, n, B,
                  kv->max_seq_len);
    a.n_old[b] = n;
    if (B > 0) {
      const int touched = (n + B - 1) / v.page_size - n / v.page_size + 1;
      max_touched = touched > max_touched ? touched : max_touched;
    }
  }
  if (B == 0) return FB_OK;
  a.k_in = k_in;
  a.v_in = v_in;
  a.k = const_cast<void*>(kv->k);
  a.v = const_cast<void*>(kv->v);
  a.page_table = kv->page_table;
  a.seq_len = const_cast<int32_t*>(kv->seq_len);
  a.pmin = page_min;
  a.pmax = page_max;
  a.n_slots = kv->n_slots;
  a.batch = kv->batch;
  a.B = B;
  a.Hkv = kv->n_heads_kv;
  a.page_size = v.page_size;
  a.max_pages = v.max_pages;
  a.max_seq_len = kv->max_seq_len;
  const dim3 grid(max_touched, kv->n_heads_kv, kv->batch);
  if (grid.y > 65535) return fail(FB_ERR_SHAPE, "too many kv heads");
  if (!aligned16(kv->k) || !aligned16(kv->v)) return fail(FB_ERR_ALIGN, "k / v not 16-byte aligned");
  // shared memory: the new K rows of one page
  const int sm = v.page_size * v.D * (int)elem_size(kv->dtype);
  if (sm > 160 * 1024) return fail(FB_ERR_SHAPE, "page_size %d too large for the commit", v.page_size);
#define FB_COMMIT(TT, DD)                                                          \
  do {                                                                             \
    auto kfn = block_commit_kernel<TT, DD>;                                        \
    if (int rc_ = set_smem_once((const void*)kfn, sm)) return rc_;                \
    kfn<<<grid, kCommitThreads, sm, stream>>>(a);                                  \
  } while (0)
  if (kv->dtype == FB_BF16) {
    if (v.D == 128) FB_COMMIT(__nv_bfloat16, 128); else FB_COMMIT(__nv_bfloat16, 64);
  } else {
    if (v.D == 128) FB_COMMIT(float, 128); else FB_COMMIT(float, 64);
  }
#undef FB_COMMIT
  return check_launch("block commit kernel");
}

size_t fb_workspace_size(const fb_kv* kv, int32_t block, int32_t n_heads_q, int32_t n_active,
                         int32_t topk_pages, int32_t num_sms) {
  if (!kv || block <= 0 || n_heads_q <= 0 || kv->n_heads_kv <= 0 || n_heads_q % kv->n_heads_kv ||
      kv->batch <= 0 || kv->max_seq_len < 0 || kv->page_size <= 0)
    return 0;
  // shapes no call accepts have no workspace size either
  if ((kv->head_dim != 64 && kv->head_dim != 128) || !pow2(kv->page_size) || kv->page_size < 16 ||
      (kv->dtype != FB_BF16 && kv->dtype != FB_F32) || n_active < 0 || topk_pages < 0)
    return 0;
  if (num_sms <= 0) num_sms = sm_count();
  if (num_sms <= 0) return 0;
  return ws_layout(kv, block, n_heads_q, n_active, topk_pages, num_sms).total;
}

size_t fb_workspace_page_scores(const fb_kv* kv, int32_t block, int32_t n_heads_q,
                                int32_t n_active, int32_t topk_pages, int32_t num_sms) {
  if (n_active <= 0 || topk_pages <= 0) return 0;
  if (fb_workspace_size(kv, block, n_heads_q, n_active, topk_pages, num_sms) == 0) return 0;
  if (num_sms <= 0) num_sms = sm_count();
  return ws_layout(kv, block, n_heads_q, n_active, topk_pages, num_sms).scores;
}

int fb_prefix_attn(const void* q, int32_t B, int32_t n_heads_q, float scale, const fb_kv* kv,
                   const uint8_t* head_mask, float* a_out, float* l_out, void* workspace,
                   size_t workspace_bytes, cudaStream_t stream) {
  int rc = validate_kv(kv);
  if (rc) return rc;
  rc = validate_q(q, B, n_heads_q, kv);
  if (rc) return rc;
  if (!a_out || !l_out) return fail(FB_ERR_ARG, "a_out / l_out is NULL");
  PartialCall c{};
  c.q = q;
  c.B = B;
  c.Hq = n_heads_q;
  c.scale = scale;
  c.kv = kv;
  c.head_mask = head_mask;
  c.a_out = a_out;
  c.l_out = l_out;
  c.ws = workspace;
  c.ws_bytes = workspace_bytes;
  c.num_sms = sm_count();
  return launch_partial(c, stream);
}

int fb_block_attn(const void* q, const void* k_in, const void* v_in, int32_t batch, int32_t B,
                  int32_t n_heads_q, int32_t n_heads_kv, int32_t head_dim, float scale,
                  fb_dtype dtype, float* a_in, float* l_in, cudaStream_t stream) {
  return block_attn_impl(q, k_in, v_in, batch, B, n_heads_q, n_heads_kv, head_dim, scale, dtype,
                         a_in, l_in, stream);
}

int fb_merge(const float* a_out, const float* l_out, const float* a_in, const float* l_in,
             int64_t rows, int32_t head_dim, float* a_full, float* l_full, cudaStream_t stream) {
  if (!a_out || !l_out || !a_in || !l_in || !a_full) return fail(FB_ERR_ARG, "NULL argument");
  if (rows < 0) return fail(FB_ERR_ARG, "rows < 0");
  if (head_dim != 64 && head_dim != 128) return fail(FB_ERR_SHAPE, "head_dim must be 64 or 128");
  return merge_launch(a_out, l_out, a_in, l_in, rows, head_dim, a_full, l_full, stream);
}

int fb_page_summary(const fb_kv* kv, void* page_min, void* page_max, cudaStream_t stream) {
  int rc = validate_kv(kv);
  if (rc) return rc;
  if (!page_min || !page_max) return fail(FB_ERR_ARG, "page_min / page_max is NULL");
  const KvView v = kv_view(kv);
  const long long warps = (long long)v.batch * v.max_pages * v.Hkv;
  if (warps == 0) return FB_OK;
  const int blocks = ceil_div(warps * 32, 256);
  if (kv->dtype == FB_BF16) {
    auto* mn = static_cast<__nv_bfloat16*>(page_min);
    auto* mx = static_cast<__nv_bfloat16*>(page_max);
    if (v.D == 128)
      page_summary_kernel<__nv_bfloat16, 128><<<blocks, 256, 0, stream>>>(v, mn, mx);
    else
      page_summary_kernel<__nv_bfloat16, 64><<<blocks, 256, 0, stream>>>(v, mn, mx);
  } else {
    auto* mn = static_cast<float*>(page_min);
    auto* mx = static_cast<float*>(page_max);
    if (v.D == 128)
      page_summary_kernel<float, 128><<<blocks, 256, 0, stream>>>(v, mn, mx);
    else
      page_summary_kernel<float, 64><<<blocks, 256, 0, stream>>>(v, mn, mx);
  }
  return check_launch("page summary kernel");
}

int losa_select(const void* q_cur, const void* q_prev, int32_t B, int32_t n_heads_q,
                const void* page_min, const void* page_max, const fb_kv* kv, int32_t n_active,
                int32_t topk_pages, int32_t* active_rows, float* row_scores,
                uint32_t* union_bitmap, int32_t* union_list, int32_t* union_count,
                void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  int rc = validate_kv(kv);
  if (rc) return rc;
  rc = validate_q(q_cur, B, n_heads_q, kv);
  if (rc) return rc;
  if (!q_prev || !page_min || !page_max || !active_rows || !union_bitmap || !union_list ||
      !union_count)
    return fail(FB_ERR_ARG, "NULL argument");
  if (n_active < 0 || topk_pages < 0) return fail(FB_ERR_ARG, "n_active / topk_pages < 0");
  if (!aligned16(page_min) || !aligned16(page_max) || !aligned16(q_prev))
    return fail(FB_ERR_ALIGN, "page summaries / q_prev not 16-byte aligned");
  const KvView v = kv_view(kv);
  const int D = v.D, Hq = n_heads_q, G = Hq / v.Hkv;
  const int na = n_active < B ? n_active : B;
  const int words = ceil_div(v.max_pages, 32);
  if (v.max_pages > 32768) return fail(FB_ERR_SHAPE, "LoSA selection supports <= 32768 pages");
  if (Hq * D > 16384) return fail(FB_ERR_SHAPE, "LoSA selection supports n_heads_q * d <= 16384");
  const int num_sms = sm_count();
  const WsLayout w = ws_layout(kv, B, Hq, n_active, topk_pages, num_sms);
  if (!workspace || workspace_bytes < w.total)
    return fail(FB_ERR_WORKSPACE, "workspace too small: need %zu, have %zu", w.total,
                workspace_bytes);
  char* ws = static_cast<char*>(workspace);
  float* page_scores = reinterpret_cast<float*>(ws + w.scores);
  int* tickets = reinterpret_cast<int*>(ws + w.tickets);
  float* rs = row_scores
                  ? row_scores
                  : reinterpret_cast<float*>(ws + w.scores +
                                             round_up((size_t)kv->batch * na * Hq * v.max_pages * 4,
                                                      256));
  const int N = Hq * D, N2 = next_pow2(N);
  if (na == 0) {
    // no active rows: an empty union (the bitmap and counts still get written)
    cudaMemsetAsync(union_bitmap, 0, (size_t)kv->batch * v.Hkv * words * 4, stream);
    cudaMemsetAsync(union_count, 0, (size_t)kv->batch * v.Hkv * 4, stream);
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? FB_OK : fail(FB_ERR_CUDA, "losa_select memset: %s", cudaGetErrorString(e));
  }
  const dim3 g1(B, kv->batch);
  if (N2 >= 256 && N2 <= 256 * 32) {
    // register tree (E elements per thread)
#define FB_LOC(TT, EE)                                                                         \
  launch_pdl(locality_score_reg_kernel<TT, EE>, g1, dim3(256), 0, stream,                     \
             static_cast<const TT*>(q_cur), static_cast<const TT*>(q_prev), B, N, rs)
#define FB_LOC_E(TT)          \
  switch (N2 / 256) {         \
    case 1: FB_LOC(TT, 1); break;   \
    case 2: FB_LOC(TT, 2); break;   \
    case 4: FB_LOC(TT, 4); break;   \
    case 8: FB_LOC(TT, 8); break;   \
    case 16: FB_LOC(TT, 16); break; \
    default: FB_LOC(TT, 32); break; \
  }
    if (kv->dtype == FB_BF16) {
      FB_LOC_E(__nv_bfloat16)
    } else {
      FB_LOC_E(float)
    }
#undef FB_LOC_E
#undef FB_LOC
  } else {
    rc = kv->dtype == FB_BF16
             ? set_smem_once((const void*)locality_score_kernel<__nv_bfloat16>, N2 * 4)
             : set_smem_once((const void*)locality_score_kernel<float>, N2 * 4);
    if (rc) return rc;
    if (kv->dtype == FB_BF16)
      launch_pdl(locality_score_kernel<__nv_bfloat16>, g1, dim3(256), N2 * 4, stream,
                 static_cast<const __nv_bfloat16*>(q_cur),
                 static_cast<const __nv_bfloat16*>(q_prev), B, N, N2, rs);
    else
      launch_pdl(locality_score_kernel<float>, g1, dim3(256), N2 * 4, stream,
                 static_cast<const float*>(q_cur), static_cast<const float*>(q_prev), B, N, N2,
                 rs);
  }
  rc = check_launch("locality score kernel");
  if (rc) return rc;
  // Up to 32 active rows are picked inside the page scorer (every CTA of a
  // sequence from the same locality scores); more take the rank kernel.
  const bool pick_in_scorer = na <= 32;
  if (!pick_in_scorer) {
    launch_pdl(active_rows_kernel, dim3(kv->batch), dim3(256), B * 4, stream, (const float*)rs,
               B, na, active_rows);
    rc = check_launch("active rows kernel");
    if (rc) return rc;
  }
  const int32_t* act_in = pick_in_scorer ? nullptr : active_rows;
  const float* rs_in = pick_in_scorer ? rs : nullptr;
  if (kv->dtype == FB_BF16) {
    int tpc;
    const int psm = page_score_cols_smem(na * G, D, false) + (pick_in_scorer ? B * 4 : 0);
    const dim3 g2 = page_cols_grid(v, num_sms, psm, tpc);
    const bool one = na * G <= kPcRows;
    auto kfn = D == 128 ? (one ? page_score_cols_kernel<128, kPcRowsOnePass>
                               : page_score_cols_kernel<128, kPcRowsMulti>)
                        : (one ? page_score_cols_kernel<64, kPcRowsOnePass>
                               : page_score_cols_kernel<64, kPcRowsMulti>);
    if ((rc = set_smem_once((const void*)kfn, psm))) return rc;
    launch_pdl(kfn, g2, dim3(kPcThreads), psm, stream, static_cast<const __nv_bfloat16*>(q_cur),
               act_in, rs_in, active_rows, B, Hq, G, na,
               static_cast<const __nv_bfloat16*>(page_min),
               static_cast<const __nv_bfloat16*>(page_max), v, page_scores, union_bitmap, words,
               tickets, tpc);
  } else {
    int cpc;
    const int psm = page_score_smem(na * G, D) + (pick_in_scorer ? B * 4 : 0);
    const dim3 g2 = page_score_grid(v, num_sms, psm, cpc);
    auto kfn = D == 128 ? page_score_kernel<float, 128> : page_score_kernel<float, 64>;
    if ((rc = set_smem_once((const void*)kfn, psm))) return rc;
    launch_pdl(kfn, g2, dim3(256), psm, stream, static_cast<const float*>(q_cur), act_in, rs_in,
               active_rows, B, Hq, G, na, static_cast<const float*>(page_min),
               static_cast<const float*>(page_max), v, page_scores, union_bitmap, words, tickets,
               cpc);
  }
  rc = check_launch("page score kernel");
  if (rc) return rc;
  // top-k per (active row, q head); the last CTA of each kv head compacts the union
  const int ksm = (v.max_pages + words) * 4;
  if ((rc = set_smem_once((const void*)topk_pages_kernel, ksm))) return rc;
  launch_pdl(topk_pages_kernel, dim3(na * Hq, kv->batch), dim3(kTopkThreads), ksm, stream,
             (const float*)page_scores, v, Hq, G, na, topk_pages, union_bitmap, words, union_list,
             union_count, v.max_pages, tickets);
  return check_launch("top-k pages kernel");
}

int losa_gather(const void* q, int32_t B, int32_t n_heads_q, const int32_t* active_rows,
                int32_t n_active, const int32_t* union_list, const int32_t* union_count,
                int32_t max_union, const fb_kv* kv, float scale, float* a_out, float* l_out,
                void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  int rc = validate_kv(kv);
  if (rc) return rc;
  rc = validate_q(q, B, n_heads_q, kv);
  if (rc) return rc;
  if (!a_out || !l_out || !union_list || !union_count || (n_active > 0 && !active_rows))
    return fail(FB_ERR_ARG, "NULL argument");
  const int na = n_active < B ? n_active : B;
  if (na <= 0) return FB_OK;
  const KvView v = kv_view(kv);
  PartialCall c{};
  c.q = q;
  c.B = B;
  c.Hq = n_heads_q;
  c.scale = scale;
  c.kv = kv;
  c.row_list = active_rows;
  c.n_list = na;
  c.page_list = union_list;
  c.page_count = union_count;
  c.page_list_stride = v.max_pages;
  c.max_list_entries = (max_union > 0 && max_union < v.max_pages) ? max_union : v.max_pages;
  c.a_out = a_out;
  c.l_out = l_out;
  c.ws = workspace;
  c.ws_bytes = workspace_bytes;
  c.num_sms = sm_count();
  return launch_partial(c, stream);
}

// One denoise step (fb_step); with cu != NULL the block rows are packed
// (fb_step_varlen): B is the most rows any sequence has, total the packed rows.
static int step_impl(const fb_policy* policy, fb_cache* cache, const void* q, const void* k_in,
                     const void* v_in, int32_t B, int32_t n_heads_q, const fb_kv* prefix,
                     const void* page_min, const void* page_max, const int32_t* m_updated,
                     float* a_full, float* l_full, void* workspace, size_t workspace_bytes,
                     const int32_t* cu, int32_t total, cudaStream_t stream) {
  if (!policy || !cache) return fail(FB_ERR_ARG, "policy / cache is NULL");
  if (cu && policy->mode != FB_THRESHOLD)
    return fail(FB_ERR_ARG, "packed rows support the threshold controller only");
  int rc = validate_kv(prefix);
  if (rc) return rc;
  rc = validate_q(q, B, n_heads_q, prefix);
  if (rc) return rc;
  if (!k_in || !v_in || !a_full || !cache->a_out || !cache->l_out)
    return fail(FB_ERR_ARG, "NULL argument");
  const int batch = prefix->batch, Hq = n_heads_q, Hkv = prefix->n_heads_kv, D = prefix->head_dim;
  const int s = cache->step;
  const int num_sms = sm_count();
  const bool sr = policy->mode == FB_SPARSE_RESIDUAL;
  const int na = policy->mode == FB_LOSA ? policy->n_active : (sr ? B : 0);
  const int tk = policy->mode == FB_LOSA ? policy->topk_pages : (sr ? logical_pages(prefix) : 0);
  const WsLayout w = ws_layout(prefix, B, Hq, na, tk, num_sms);
  if (!workspace || workspace_bytes < w.total)
    return fail(FB_ERR_WORKSPACE, "workspace too small: need %zu, have %zu", w.total,
                workspace_bytes);
  char* ws = static_cast<char*>(workspace);
  PartialCall c{};
  c.q = q;
  c.B = B;
  c.Hq = Hq;
  c.scale = policy->scale;
  c.kv = prefix;
  c.a_out = cache->a_out;
  c.l_out = cache->l_out;
  c.ws = workspace;
  c.ws_bytes = workspace_bytes;
  c.ws_offset = w.part;
  c.num_sms = num_sms;
  c.q_cu = cu;
  c.q_total = total;

  if (policy->mode == FB_THRESHOLD) {
    unsigned long long bits[4] = {0, 0, 0, 0};
    int n_rec = 0;
    for (int b = 0; b < batch; ++b) {
      const bool rec = s == 0 || policy->tau <= 0 || (m_updated && m_updated[b] >= policy->tau);
      if (rec) {
        bits[b >> 6] |= 1ull << (b & 63);
        ++n_rec;
      }
    }
    cache->recomputed = n_rec;
    if (n_rec > 0) {
      c.seq_bits = n_rec < batch ? bits : nullptr;
      rc = launch_partial(c, stream);
      if (rc) return rc;
    }
  } else if (policy->mode == FB_PER_HEAD) {
    if (!cache->head_mask || !cache->a_out_prev || !cache->head_cos)
      return fail(FB_ERR_ARG, "PER_HEAD needs head_mask, a_out_prev and head_cos");
    if (s == 0) {
      if (cudaMemsetAsync(cache->head_mask, 1, (size_t)batch * Hq, stream) != cudaSuccess)
        return fail(FB_ERR_CUDA, "head mask reset failed");
    }
    c.head_mask = cache->head_mask;
    c.a_prev = cache->a_out_prev;
    rc = launch_partial(c, stream);
    if (rc) return rc;
    if (s >= 1) {
      const int N = B * D, P = next_pow2(N);
      if (P > kCosT1Max * kCosEMax) return fail(FB_ERR_SHAPE, "B * d too large for the cosine");
      const int T1 = P < kCosT1Max ? P : kCosT1Max, E = P / T1;
      double* part = reinterpret_cast<double*>(ws + w.cos);
      head_cos_stage1<<<dim3(ceil_div(T1, 256), batch * Hq), 256, 0, stream>>>(
          cache->a_out, cache->a_out_prev, cache->head_mask, B, Hq, D, N, T1, E, part);
      rc = check_launch("cosine stage 1");
      if (rc) return rc;
      head_cos_stage2<<<batch * Hq, 1024, 0, stream>>>(part, T1, policy->gamma, cache->head_mask,
                                                      cache->head_cos);
      rc = check_launch("cosine stage 2");
      if (rc) return rc;
    }
  } else if (sr) {
    if (!page_min || !page_max || !cache->union_bitmap || !cache->union_list ||
        !cache->union_count || !cache->comp_list || !cache->comp_count || !cache->a_res ||
        !cache->l_res)
      return fail(FB_ERR_ARG, "SPARSE_RESIDUAL needs the page summaries, the selection and "
                              "complement buffers and a_res / l_res");
    if (policy->topk_pages < 0) return fail(FB_ERR_ARG, "topk_pages < 0");
    bool refresh = s == 0 || policy->tau <= 0;
    for (int b = 0; b < batch && !refresh; ++b)
      refresh = m_updated && m_updated[b] >= policy->tau;
    cache->recomputed = refresh ? batch : 0;
    const int np = logical_pages(prefix);
    if (refresh) {
      rc = sr_select(q, B, Hq, page_min, page_max, prefix, policy->topk_pages,
                     cache->union_bitmap, cache->union_list, cache->union_count, cache->comp_list,
                     cache->comp_count, reinterpret_cast<float*>(ws + w.scores),
                     reinterpret_cast<int*>(ws + w.tickets), stream);
      if (rc) return rc;
      PartialCall cr = c;  // residual: every row over the unselected pages
      cr.page_list = cache->comp_list;
      cr.page_count = cache->comp_count;
      cr.page_list_stride = np;
      cr.max_list_entries = np;
      cr.a_out = cache->a_res;
      cr.l_out = cache->l_res;
      rc = launch_partial(cr, stream);
      if (rc) return rc;
    }
    PartialCall cs = c;  // fresh sparse partial over the selected pages, merged with the residual
    cs.page_list = cache->union_list;
    cs.page_count = cache->union_count;
    cs.page_list_stride = np;
    cs.max_list_entries = policy->topk_pages < np ? policy->topk_pages : np;
    cs.mrg_a = cache->a_res;
    cs.mrg_l = cache->l_res;
    rc = launch_partial(cs, stream);
    if (rc) return rc;
  } else if (policy->mode == FB_LOSA) {
    if (!cache->q_prev || !cache->active_rows || !cache->union_bitmap || !cache->union_list ||
        !cache->union_count)
      return fail(FB_ERR_ARG, "LOSA needs q_prev, active_rows and the union buffers");
    if (s == 0) {
      rc = launch_partial(c, stream);
      if (rc) return rc;
    } else {
      rc = losa_select(q, cache->q_prev, B, Hq, page_min, page_max, prefix, policy->n_active,
                       policy->topk_pages, cache->active_rows, cache->row_scores,
                       cache->union_bitmap, cache->union_list, cache->union_count, workspace,
                       workspace_bytes, stream);
      if (rc) return rc;
      const int na_c = policy->n_active < B ? policy->n_active : B;
      rc = losa_gather(q, B, Hq, cache->active_rows, policy->n_active, cache->union_list,
                       cache->union_count,
                       max_union_entries(prefix, Hq / Hkv, na_c, policy->topk_pages), prefix,
                       policy->scale, cache->a_out, cache->l_out, workspace, workspace_bytes,
                       stream);
      if (rc) return rc;
    }
    const size_t qbytes = (size_t)batch * B * Hq * D * elem_size(prefix->dtype);
    if (cudaMemcpyAsync(cache->q_prev, q, qbytes, cudaMemcpyDeviceToDevice, stream) != cudaSuccess)
      return fail(FB_ERR_CUDA, "q_prev copy failed");
  } else {
    return fail(FB_ERR_ARG, "unknown mode");
  }
  // block-internal partial and the FlashBlock merge with the cached
  // block-external partial in one kernel: A_full directly
  float* lf = l_full ? l_full : reinterpret_cast<float*>(ws + w.l_in);
  // (the in-block call may use the split-partial region of the workspace: the
  // prefix partial's combine, earlier on the stream, is done with it)
  rc = block_attn_impl(q, k_in, v_in, batch, B, Hq, Hkv, D, policy->scale, prefix->dtype, a_full,
                       lf, stream, cache->a_out, cache->l_out, cu, total, workspace, w.scores,
                       w.part);
  if (rc) return rc;
  cache->step = s + 1;
  return FB_OK;
}

int fb_step(const fb_policy* policy, fb_cache* cache, const void* q, const void* k_in,
            const void* v_in, int32_t B, int32_t n_heads_q, const fb_kv* prefix,
            const void* page_min, const void* page_max, const int32_t* m_updated, float* a_full,
            float* l_full, void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  return step_impl(policy, cache, q, k_in, v_in, B, n_heads_q, prefix, page_min, page_max,
                   m_updated, a_full, l_full, workspace, workspace_bytes, nullptr, 0, stream);
}

// Host checks shared by the packed-row entry points.
static int validate_packed(const int32_t* cu_rows, int32_t max_rows, int32_t total_rows) {
  if (!cu_rows) return fail(FB_ERR_ARG, "cu_rows is NULL");
  if (max_rows <= 0) return fail(FB_ERR_ARG, "max_rows must be positive");
  if (total_rows < 0) return fail(FB_ERR_ARG, "total_rows must be >= 0");
  return FB_OK;
}

int fb_prefix_attn_varlen(const void* q, const int32_t* cu_rows, int32_t max_rows,
                          int32_t total_rows, int32_t n_heads_q, float scale, const fb_kv* kv,
                          float* a_out, float* l_out, void* workspace, size_t workspace_bytes,
                          cudaStream_t stream) {
  int rc = validate_kv(kv);
  if (rc) return rc;
  if ((rc = validate_packed(cu_rows, max_rows, total_rows))) return rc;
  rc = validate_q(q, max_rows, n_heads_q, kv);
  if (rc) return rc;
  if (!a_out || !l_out) return fail(FB_ERR_ARG, "a_out / l_out is NULL");
  if (total_rows == 0) return FB_OK;
  PartialCall c{};
  c.q = q;
  c.B = max_rows;
  c.Hq = n_heads_q;
  c.scale = scale;
  c.kv = kv;
  c.a_out = a_out;
  c.l_out = l_out;
  c.ws = workspace;
  c.ws_bytes = workspace_bytes;
  c.num_sms = sm_count();
  c.q_cu = cu_rows;
  c.q_total = total_rows;
  return launch_partial(c, stream);
}

int fb_block_attn_varlen(const void* q, const void* k_in, const void* v_in,
                         const int32_t* cu_rows, int32_t batch, int32_t max_rows,
                         int32_t total_rows, int32_t n_heads_q, int32_t n_heads_kv,
                         int32_t head_dim, float scale, fb_dtype dtype, float* a_in, float* l_in,
                         cudaStream_t stream) {
  int rc = validate_packed(cu_rows, max_rows, total_rows);
  if (rc) return rc;
  if (!k_in || !v_in) return fail(FB_ERR_ARG, "k_in / v_in is NULL");
  if (!aligned16(k_in) || !aligned16(v_in)) return fail(FB_ERR_ALIGN, "k_in / v_in not 16-byte aligned");
  return block_attn_impl(q, k_in, v_in, batch, max_rows, n_heads_q, n_heads_kv, head_dim, scale,
                         dtype, a_in, l_in, stream, nullptr, nullptr, cu_rows, total_rows);
}

int fb_step_varlen(const fb_policy* policy, fb_cache* cache, const void* q, const void* k_in,
                   const void* v_in, const int32_t* cu_rows, int32_t max_rows,
                   int32_t total_rows, int32_t n_heads_q, const fb_kv* prefix,
                   const int32_t* m_updated, float* a_full, float* l_full, void* workspace,
                   size_t workspace_bytes, cudaStream_t stream) {
  int rc = validate_packed(cu_rows, max_rows, total_rows);
  if (rc) return rc;
  if (total_rows == 0) {
    if (cache) cache->step += 1;
    return FB_OK;
  }
  return step_impl(policy, cache, q, k_in, v_in, max_rows, n_heads_q, prefix, nullptr, nullptr,
                   m_updated, a_full, l_full, workspace, workspace_bytes, cu_rows, total_rows,
                   stream);
}

// Unique id of the calling thread's current context (false if none is current
// or the driver has no id query). A context created after cudaDeviceReset may
// reuse the handle of the one it replaced, so the id, not the handle, tells
// whether a remembered device address still belongs to the live context.
static bool current_context_id(unsigned long long* id) {
  static PFN_cuCtxGetCurrent_v4000 get_cur = nullptr;
  static PFN_cuCtxGetId_v12000 get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_cur = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(p);
  });
  CUcontext ctx = nullptr;
  if (!get_cur || !get_id || get_cur(&ctx) != CUDA_SUCCESS || !ctx) return false;
  return get_id(ctx, id) == CUDA_SUCCESS;
}

// Device address of g_fb_noalloc_scratch on the current device. It is looked up
// with cudaGetSymbolAddress on the first call made with that device current and
// remembered together with the context it belongs to; a call that finds another
// context current (the device was reset and the module loaded again) looks it
// up afresh instead of handing a stale address to the kernels.
static int noalloc_scratch(void** out) {
  struct Entry {
    void* addr;
    unsigned long long ctx;
  };
  static std::mutex mu;
  static Entry seen[256] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 256)
    return fail(FB_ERR_CUDA, "fb_prefix_attn_noalloc: no current device");
  std::lock_guard<std::mutex> lock(mu);
  unsigned long long ctx = 0;
  const bool have_ctx = current_context_id(&ctx);
  if (!seen[dev].addr || !have_ctx || seen[dev].ctx != ctx) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_fb_noalloc_scratch);
    if (e != cudaSuccess || !p)
      return fail(FB_ERR_CUDA, "fb_prefix_attn_noalloc: cudaGetSymbolAddress failed: %s",
                  cudaGetErrorString(e));
    // the lookup made the device's context current on this thread if it was not
    seen[dev].addr = p;
    seen[dev].ctx = current_context_id(&ctx) ? ctx : 0;
  }
  *out = seen[dev].addr;
  return FB_OK;
}

int fb_prefix_attn_noalloc(const void* q, int32_t B, int32_t n_heads_q, float scale,
                           const fb_kv* kv, const uint8_t* head_mask, float* a_out, float* l_out,
                           cudaStream_t stream) {
  int rc = validate_kv(kv);
  if (rc) return rc;
  rc = validate_q(q, B, n_heads_q, kv);
  if (rc) return rc;
  if (!a_out || !l_out) return fail(FB_ERR_ARG, "a_out / l_out is NULL");
  if ((rc = validate_scale(scale))) return rc;
  const int num_sms = sm_count();
  const int R = B * (n_heads_q / kv->n_heads_kv);
  const size_t need = partial_ws_bytes(kv->dtype, kv->batch, kv->n_heads_kv, R, kv->head_dim,
                                       ceil_div(kv->max_seq_len, kTK), num_sms);
  if (need > (size_t)FB_NOALLOC_SCRATCH_BYTES)
    return fail(FB_ERR_WORKSPACE,
                "fb_prefix_attn_noalloc: these shapes need %zu bytes of scratch but the static "
                "buffer holds %zu; use fb_prefix_attn with a workspace",
                need, (size_t)FB_NOALLOC_SCRATCH_BYTES);
  void* scratch = nullptr;
  rc = noalloc_scratch(&scratch);
  if (rc) return rc;
  // Nothing in the scratch has to start at zero: every split of every row writes
  // its partial and normaliser (an empty split: zeros and -inf) before the
  // combine reads them, and the combine gives an empty split no weight.
  PartialCall c{};
  c.q = q;
  c.B = B;
  c.Hq = n_heads_q;
  c.scale = scale;
  c.kv = kv;
  c.head_mask = head_mask;
  c.a_out = a_out;
  c.l_out = l_out;
  c.ws = scratch;
  c.ws_bytes = FB_NOALLOC_SCRATCH_BYTES;
  c.num_sms = num_sms;
  return launch_partial(c, stream);
}

}  // extern "C"
