// qsa_api.cu -- C ABI of libqsa.so: argument checks, workspace layout, TMA descriptors and
// kernel launches for QSA prefill, append and decode on sm_100a.  The declarations and the
// contract of every entry point are in include/qsa.h.
#include <algorithm>
#include <atomic>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <vector>

#include "../../include/qsa.h"
#include "qsa_attn.cuh"
#include "qsa_common.cuh"
#include "qsa_gdn.cuh"
#include "qsa_misc.cuh"
#include "qsa_score.cuh"

using namespace qsa;

namespace {

constexpr int kVersion = 100;   // 0.1.0
constexpr int kDefaultRowsPerTile = 10;
constexpr int kDefaultScoreChunkRows = 16384;
constexpr int kTopkCandCap = 4096;      // per-row candidates of the score-row top-k
constexpr int kCandCap = 16384;         // decode top-k candidates per row
constexpr int kNumSMsFallback = 148;

// ---- driver entry point for tensor-map encoding (no link-time libcuda dependency) ----
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static std::once_flag once;
  static EncodeTiledFn fn = nullptr;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

int num_sms() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return kNumSMsFallback;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
    return kNumSMsFallback;
  return n;
}

// bf16 tensor map, 128-byte swizzle, inner box of 64 elements (128 bytes).
bool make_tmap(CUtensorMap* m, const void* base, int rank, const uint64_t* dims,
               const uint64_t* strides_bytes, const uint32_t* box) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t gd[5];
  cuuint64_t gs[4];
  cuuint32_t bd[5], es[5];
  for (int i = 0; i < rank; ++i) {
    gd[i] = dims[i];
    bd[i] = box[i];
    es[i] = 1;
  }
  for (int i = 0; i < rank - 1; ++i) gs[i] = strides_bytes[i];
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(base), gd, gs, bd,
                  es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// ---- workspace carving ---------------------------------------------------------------
struct Carver {
  size_t off = QSA_WS_HEADER_BYTES;
  size_t take(size_t bytes) {
    const size_t o = off;
    off = round_up(off + bytes, 256);
    return o;
  }
};

struct PrefillGeom {
  int64_t T = 0;
  int32_t max_len = 0;
  int64_t total_blocks = 0;
  int32_t max_nc = 0;
  int64_t ld = 0;
  int32_t score_tiles = 0;
  int32_t attn_tiles = 0;
  int32_t R = kDefaultRowsPerTile;
  int32_t topk = 512;
  int32_t chunk_rows = kDefaultScoreChunkRows;
  int32_t fault = 0;   // qsa_params.debug_fault
  bool fused = false;  // qsa_params.select_mode 1 applies: the indexer finds each row's threshold bin
  PlanLayout pl;
  int32_t max_words = 1;
  // workspace offsets
  size_t o_meta = 0, o_kbar = 0, o_nc = 0, o_scores = 0, o_rinfo = 0, o_idx = 0, o_cnt = 0,
         o_plan = 0, total = 0;
};

qsa_status prefill_geom(const int32_t* h_cu, int32_t num_seqs, const qsa_params& p,
                        PrefillGeom* g) {
  if (!h_cu || num_seqs <= 0) return QSA_ERR_INVALID_ARG;
  if (p.topk_blocks < 1 || p.topk_blocks > QSA_MAX_TOPK) return QSA_ERR_INVALID_ARG;
  if (p.debug_fault != 0 && p.debug_fault != 1) return QSA_ERR_INVALID_ARG;
  if (p.select_mode != 0 && p.select_mode != 1) return QSA_ERR_INVALID_ARG;
  if (h_cu[0] != 0) return QSA_ERR_INVALID_ARG;
  g->fault = p.debug_fault;
  g->R = p.rows_per_tile > 0 ? p.rows_per_tile : kDefaultRowsPerTile;
  if (g->R < 1 || g->R > 10) return QSA_ERR_INVALID_ARG;
  g->topk = p.topk_blocks;
  g->chunk_rows = p.score_chunk_rows > 0 ? p.score_chunk_rows : kDefaultScoreChunkRows;
  if (g->chunk_rows < 16) g->chunk_rows = 16;
  int64_t T = 0, blocks = 0;
  int32_t max_len = 0;
  int64_t st = 0, at = 0;
  for (int s = 0; s < num_seqs; ++s) {
    const int64_t L = static_cast<int64_t>(h_cu[s + 1]) - h_cu[s];
    if (L < 1 || L > QSA_MAX_SEQ_LEN) return QSA_ERR_INVALID_ARG;
    T += L;
    blocks += L / 4;
    max_len = std::max<int32_t>(max_len, static_cast<int32_t>(L));
    st += (L + 15) / 16;
    at += (L + g->R - 1) / g->R;
  }
  if (T > (int64_t(1) << 26)) return QSA_ERR_UNSUPPORTED;
  g->T = T;
  g->max_len = max_len;
  g->total_blocks = blocks;
  g->max_nc = (max_len - 1) / 4;
  // the indexer's per-row histograms count in 16 bits: rows of fewer than 65,536 candidates
  g->fused = p.select_mode == 1 && g->max_nc < 65536;
  g->ld = std::max<int64_t>(4, round_up(std::max(g->max_nc, 1), 4));
  g->score_tiles = static_cast<int32_t>(st);
  g->attn_tiles = static_cast<int32_t>(at);
  g->pl = make_plan_layout(g->R, g->topk);
  g->max_words = (max_len - 1) / 4 / 32 + 1;
  Carver c;
  g->o_meta = c.take(sizeof(SeqMeta) * (num_seqs + 1));
  g->o_kbar = c.take(static_cast<size_t>(std::max<int64_t>(blocks, 1)) * 64 * 2);
  g->o_nc = c.take(static_cast<size_t>(T) * 4);
  const int64_t rows = std::min<int64_t>(T, g->chunk_rows + 16);
  g->o_scores = c.take(static_cast<size_t>(rows) * g->ld * 4);
  if (g->fused) g->o_rinfo = c.take(static_cast<size_t>(rows) * 4 * 4);   // threshold bin per row
  g->o_idx = c.take(static_cast<size_t>(T) * g->topk * 4);
  g->o_cnt = c.take(static_cast<size_t>(T) * 4);
  g->o_plan = c.take(static_cast<size_t>(g->attn_tiles) * g->pl.stride * 4);
  g->total = c.off;
  return QSA_OK;
}

std::atomic<uint64_t> g_launches{0};

#define QSA_CHECK_LAUNCH()                                  \
  do {                                                      \
    g_launches.fetch_add(1, std::memory_order_relaxed);     \
    cudaError_t e_ = cudaGetLastError();                    \
    if (e_ != cudaSuccess) {                                \
      fprintf(stderr, "qsa: launch failed: %s (%s:%d)\n",  \
              cudaGetErrorString(e_), __FILE__, __LINE__);  \
      return QSA_ERR_CUDA;                                  \
    }                                                       \
  } while (0)

// Launches a kernel with programmatic stream serialization: it may start while the kernel
// before it in the stream finishes; the kernel waits (pdl_wait) before it uses its inputs.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t s, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

#define QSA_CHECK_PDL(expr)                                  \
  do {                                                       \
    g_launches.fetch_add(1, std::memory_order_relaxed);      \
    cudaError_t e_ = (expr);                                 \
    if (e_ != cudaSuccess) {                                 \
      fprintf(stderr, "qsa: launch failed: %s (%s:%d)\n",   \
              cudaGetErrorString(e_), __FILE__, __LINE__);   \
      return QSA_ERR_CUDA;                                   \
    }                                                        \
  } while (0)

template <typename K>
bool set_smem(K kernel, int bytes) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) ==
         cudaSuccess;
}

DevStatus dev_status(void* ws) { return DevStatus{reinterpret_cast<uint32_t*>(ws)}; }

// ---- launch helpers ----------------------------------------------------------------
qsa_status launch_meta(const int32_t* d_cu, int num_seqs, int R, SeqMeta* meta, DevStatus st,
                       cudaStream_t s) {
  k_seq_meta<<<1, 1024, 0, s>>>(d_cu, num_seqs, R, meta, st);
  QSA_CHECK_LAUNCH();
  return QSA_OK;
}

qsa_status launch_compress(const void* k_idx, const SeqMeta* meta, int num_seqs,
                           int64_t total_blocks, void* kbar, cudaStream_t s) {
  if (total_blocks == 0) return QSA_OK;
  const int64_t n = total_blocks * 8;
  const int threads = 256;
  const int64_t want = (n + threads - 1) / threads;
  const int grid = static_cast<int>(std::min<int64_t>(want, int64_t(num_sms()) * 16));
  k_compress<<<grid, threads, 0, s>>>(reinterpret_cast<const uint4*>(k_idx), meta, num_seqs,
                                      reinterpret_cast<uint4*>(kbar));
  QSA_CHECK_LAUNCH();
  return QSA_OK;
}

// Top-k over `rows` score rows (one CTA per row, grid-strided).
// rinfo: each row's threshold bin as the indexer found it (select_mode 1), or null.
qsa_status launch_topk(const float* scores, int64_t ld, const int32_t* n_c, int64_t rows,
                       int topk, int max_nc, int32_t* idx, int32_t* cnt, cudaStream_t s,
                       const int32_t* rinfo = nullptr) {
  if (rows <= 0) return QSA_OK;
  const int n_max = std::max(max_nc, 1);
  const int smem = kTopkSharedBytes + kTopkCandCap * 8 + 2 * ((n_max + 31) / 32) * 4;
  if (!set_smem(k_topk, smem)) return QSA_ERR_CUDA;
  const int grid = static_cast<int>(std::min<int64_t>(rows, int64_t(num_sms()) * 16));
  k_topk<<<grid, kTopkThreads, smem, s>>>(scores, ld, n_c, rows, topk, kTopkCandCap, n_max, idx,
                                          cnt, rinfo);
  QSA_CHECK_LAUNCH();
  return QSA_OK;
}

// Host-side token start of every 16-token score tile boundary, to cut score chunks.
void score_tile_token_starts(const int32_t* h_cu, int num_seqs, std::vector<int64_t>* starts) {
  starts->clear();
  for (int s = 0; s < num_seqs; ++s) {
    const int64_t L = h_cu[s + 1] - h_cu[s];
    for (int64_t p = 0; p < L; p += 16) starts->push_back(h_cu[s] + p);
  }
  starts->push_back(h_cu[num_seqs]);
}

qsa_status run_scores_and_topk(const void* q_idx, const void* w, const void* kbar,
                               const int32_t* h_cu, int num_seqs, const PrefillGeom& g,
                               unsigned char* ws, int32_t* idx, int32_t* cnt, cudaStream_t s) {
  SeqMeta* meta = reinterpret_cast<SeqMeta*>(ws + g.o_meta);
  float* scores = reinterpret_cast<float*>(ws + g.o_scores);
  const int32_t* n_c = reinterpret_cast<const int32_t*>(ws + g.o_nc);
  CUtensorMap tm_kbar, tm_qidx;
  {
    const uint64_t dims[2] = {64, static_cast<uint64_t>(std::max<int64_t>(g.total_blocks, 1))};
    const uint64_t strides[1] = {128};
    const uint32_t box[2] = {64, 128};
    if (!make_tmap(&tm_kbar, kbar, 2, dims, strides, box)) return QSA_ERR_CUDA;
  }
  {
    const uint64_t dims[2] = {64, static_cast<uint64_t>(g.T) * 16};
    const uint64_t strides[1] = {128};
    const uint32_t box[2] = {64, 256};
    if (!make_tmap(&tm_qidx, q_idx, 2, dims, strides, box)) return QSA_ERR_CUDA;
  }
  std::vector<int64_t> starts;
  score_tile_token_starts(h_cu, num_seqs, &starts);
  const int ntiles = static_cast<int>(starts.size()) - 1;
  using C = ScoreCfg<16>;
  // one CTA per SM (512 TMEM columns); select_mode 1 adds the per-row histograms
  const int smem = g.fused ? C::kSmemBytesFused : std::max(C::kSmemBytes, 116 * 1024);
  if (!set_smem(k_index_score<16>, std::max(C::kSmemBytes, 116 * 1024)) ||
      !set_smem(k_index_score<16, true>, C::kSmemBytesFused))
    return QSA_ERR_CUDA;
  int32_t* rinfo = g.fused ? reinterpret_cast<int32_t*>(ws + g.o_rinfo) : nullptr;
  int t = 0;
  while (t < ntiles) {
    int e = t + 1;
    while (e < ntiles && starts[e + 1] - starts[t] <= g.chunk_rows) ++e;
    ScoreArgs a{};
    a.meta = meta;
    a.num_seqs = num_seqs;
    a.tile_begin = t;
    a.tile_count = e - t;
    a.topk_skip = g.topk;
    a.row_begin = starts[t];
    a.w = reinterpret_cast<const __nv_bfloat16*>(w);
    a.scores = scores;
    a.ld = g.ld;
    a.rinfo = rinfo;
    a.topk = g.topk;
    a.st = dev_status(ws);
    if (g.fused) {
      k_index_score<16, true><<<e - t, C::kThreads, smem, s>>>(tm_kbar, tm_qidx, a);
    } else {
      k_index_score<16><<<e - t, C::kThreads, smem, s>>>(tm_kbar, tm_qidx, a);
    }
    QSA_CHECK_LAUNCH();
    const int64_t r0 = starts[t], r1 = starts[e];
    qsa_status st = launch_topk(scores, g.ld, n_c + r0, r1 - r0, g.topk, g.max_nc,
                                idx + r0 * g.topk, cnt + r0, s, rinfo);
    if (st != QSA_OK) return st;
    t = e;
  }
  return QSA_OK;
}

// The attention kernel sets per-warpgroup register budgets at run time.  Before its first
// launch, check that its register count per thread covers both budgets (a budget raise that
// the launch cannot supply would wait forever), and set its shared-memory size.
qsa_status prepare_attention() {
  static std::atomic<int> ready{0};   // 1: checked and usable, 2: refused
  int r = ready.load();
  if (r == 0) {
    r = 1;
    for (const void* fn : {reinterpret_cast<const void*>(k_sparse_attn<false>),
                           reinterpret_cast<const void*>(k_sparse_attn<true>),
                           reinterpret_cast<const void*>(k_sparse_attn<true, true>)}) {
      cudaFuncAttributes fa{};
      if (cudaFuncGetAttributes(&fa, fn) != cudaSuccess) return QSA_ERR_CUDA;
      if (static_cast<int64_t>(fa.numRegs) * AttnCfg::kThreads < AttnCfg::kRegsNeeded) {
        fprintf(stderr, "qsa: attention kernel built with %d registers per thread; %d needed\n",
                fa.numRegs, (AttnCfg::kRegsNeeded + AttnCfg::kThreads - 1) / AttnCfg::kThreads);
        r = 2;
      }
    }
    ready.store(r);
  }
  if (r != 1) return QSA_ERR_UNSUPPORTED;
  if (!set_smem(k_sparse_attn<false>, AttnCfg::kSmemBytes)) return QSA_ERR_CUDA;
  if (!set_smem(k_sparse_attn<true>, AttnCfg::kSmemBytes)) return QSA_ERR_CUDA;
  if (!set_smem(k_sparse_attn<true, true>, AttnCfg::kSmemBytes)) return QSA_ERR_CUDA;
  return QSA_OK;
}

qsa_status run_attention(const void* q, const void* k, const void* v, const int32_t* idx,
                         const int32_t* cnt, int num_seqs, const PrefillGeom& g,
                         unsigned char* ws, void* out, cudaStream_t s) {
  SeqMeta* meta = reinterpret_cast<SeqMeta*>(ws + g.o_meta);
  int32_t* plan = reinterpret_cast<int32_t*>(ws + g.o_plan);
  // union plans
  {
    const int mwords = g.pl.umax / 32;
    const int smem = (2 * g.max_words + g.R * mwords) * 4;
    if (!set_smem(k_attn_plan, smem)) return QSA_ERR_CUDA;
    const int grid = std::min(g.attn_tiles, num_sms() * 8);
    k_attn_plan<<<grid, kPlanThreads, smem, s>>>(idx, cnt, g.topk, meta, num_seqs, g.attn_tiles,
                                                 g.pl, g.max_words, plan, dev_status(ws));
    QSA_CHECK_LAUNCH();
  }
  AttnMaps maps;
  {
    const uint64_t dims[3] = {128, 24, static_cast<uint64_t>(g.T)};
    const uint64_t strides[2] = {256, 24 * 256};
    const uint32_t box[3] = {64, 12, static_cast<uint32_t>(g.R)};
    if (!make_tmap(&maps.q, q, 3, dims, strides, box)) return QSA_ERR_CUDA;
  }
  for (int j = 0; j < kNumBoxSizes; ++j) {
    const uint64_t dims[2] = {256, static_cast<uint64_t>(g.T)};
    const uint64_t strides[1] = {512};
    const uint32_t box[2] = {64, 4u << j};
    if (!make_tmap(&maps.k[j], k, 2, dims, strides, box)) return QSA_ERR_CUDA;
    if (!make_tmap(&maps.v[j], v, 2, dims, strides, box)) return QSA_ERR_CUDA;
  }
  {
    const qsa_status pst = prepare_attention();
    if (pst != QSA_OK) return pst;
  }
  AttnArgs a{};
  a.oob_row = static_cast<int32_t>(g.T);
  a.plan = plan;
  a.pl = g.pl;
  a.meta = meta;
  a.num_seqs = num_seqs;
  a.decode = 0;
  a.splits = 1;
  a.out = reinterpret_cast<__nv_bfloat16*>(out);
  a.st = dev_status(ws);
  a.fault_tile = g.fault == 1 ? g.attn_tiles - 1 : -1;
  dim3 grid(g.attn_tiles, 2, 1);
  k_sparse_attn<false><<<grid, AttnCfg::kThreads, AttnCfg::kSmemBytes, s>>>(maps, a);
  QSA_CHECK_LAUNCH();
  return QSA_OK;
}

qsa_status check_prefill_ptrs(std::initializer_list<const void*> ptrs) {
  for (const void* p : ptrs) {
    if (!p) return QSA_ERR_INVALID_ARG;
    if (!aligned16(p)) return QSA_ERR_ALIGNMENT;
  }
  return QSA_OK;
}

// ---- decode caches: contiguous or paged ---------------------------------------------------
// Both kinds are handled by one implementation through Paging (qsa_common.cuh): a contiguous
// cache is a pool of one page per sequence, holding its whole capacity.
struct CacheView {
  const qsa_cache* c = nullptr;   // pointers, batch, logical capacity
  Paging pg{};
  int64_t kv_rows = 0;            // rows of 128 dims in the K (and the V) pool
  int64_t kbar_rows = 0;          // rows of 64 dims in the compressed-key pool
};

CacheView contiguous_view(const qsa_cache* c) {
  CacheView v;
  v.c = c;
  v.pg = Paging{nullptr, 1, c->capacity / kBlock, c->batch};
  v.kv_rows = static_cast<int64_t>(c->batch) * 2 * c->capacity;
  v.kbar_rows = static_cast<int64_t>(c->batch) * (c->capacity / kBlock);
  return v;
}

// The base fields are checked where they are used (append, decode geometry); this checks the
// paging fields.
qsa_status paged_view(const qsa_paged_cache* pc, CacheView* v) {
  if (!pc || !pc->page_table) return QSA_ERR_INVALID_ARG;
  const qsa_cache* c = &pc->base;
  if (pc->page_tokens <= 0 || pc->page_tokens % 512 != 0 || pc->pool_pages <= 0 ||
      c->capacity <= 0 || c->capacity % pc->page_tokens != 0)
    return QSA_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(pc->page_table) % 4 != 0) return QSA_ERR_ALIGNMENT;
  const int64_t kv_rows = static_cast<int64_t>(pc->pool_pages) * 2 * pc->page_tokens;
  if (kv_rows >= 0x7fffffffll) return QSA_ERR_UNSUPPORTED;   // TMA row coordinates are int32
  v->c = c;
  v->pg = Paging{pc->page_table, c->capacity / pc->page_tokens, pc->page_tokens / kBlock,
                 pc->pool_pages};
  v->kv_rows = kv_rows;
  v->kbar_rows = static_cast<int64_t>(pc->pool_pages) * (pc->page_tokens / kBlock);
  return QSA_OK;
}

// ---- decode geometry --------------------------------------------------------------------
struct DecodeGeom {
  int32_t B = 0, cap = 0, topk = 512, max_nc = 0, splits = 4;
  int32_t cand_cap = 0;   // top-k candidates kept per row (finish kernel's shared memory)
  int64_t ld = 4;
  PlanLayout pl;
  size_t o_scores = 0, o_nc = 0, o_idx = 0, o_cnt = 0, o_plan = 0, o_po = 0, o_pm = 0, o_pl = 0,
         o_hist = 0, o_ccnt = 0, o_cand = 0, o_rinfo = 0, total = 0;
  // shared memory of k_topk_finish
  int finish_smem() const {
    return kTopkSharedBytes + cand_cap * 8 + 2 * ((std::max(max_nc, 1) + 31) / 32) * 4;
  }
};

qsa_status decode_geom(const qsa_cache* c, const qsa_params& p, DecodeGeom* g) {
  if (!c) return QSA_ERR_INVALID_ARG;
  if (c->batch <= 0 || c->capacity <= 0 || c->capacity % 4 != 0 ||
      c->capacity > QSA_MAX_SEQ_LEN)
    return QSA_ERR_INVALID_ARG;
  if (p.topk_blocks < 1 || p.topk_blocks > QSA_MAX_TOPK) return QSA_ERR_INVALID_ARG;
  if (p.debug_fault != 0) return QSA_ERR_INVALID_ARG;   // the fault hook is prefill-only
  g->B = c->batch;
  g->cap = c->capacity;
  g->topk = p.topk_blocks;
  g->max_nc = (c->capacity - 1) / 4;
  g->ld = std::max<int64_t>(4, round_up(std::max(g->max_nc, 1), 4));
  // default: as many splits as keep one wave of (sequence, KV head, split) CTAs on the SMs;
  // a CTA's fixed costs (setup, pipeline fill, partial write) favour fewer, longer CTAs
  g->splits = p.decode_splits > 0 ? p.decode_splits
                                  : std::max(1, std::min(64, num_sms() / (2 * g->B)));
  if (g->splits > 64) return QSA_ERR_INVALID_ARG;
  g->pl = make_plan_layout(1, g->topk);
  Carver cv;
  g->o_scores = cv.take(static_cast<size_t>(g->B) * g->ld * 4);
  g->o_nc = cv.take(static_cast<size_t>(g->B) * 4);
  g->o_idx = cv.take(static_cast<size_t>(g->B) * g->topk * 4);
  g->o_cnt = cv.take(static_cast<size_t>(g->B) * 4);
  g->o_plan = cv.take(static_cast<size_t>(g->B) * g->pl.stride * 4);
  const size_t parts = static_cast<size_t>(g->B) * 2 * g->splits * kGroup;
  g->o_po = cv.take(parts * kHeadDim * 4);
  g->o_pm = cv.take(parts * 4);
  g->o_pl = cv.take(parts * 4);
  // histograms and candidate counters sit back to back: one memset clears both
  g->o_hist = cv.take(static_cast<size_t>(g->B) * kTopkBins * 4 + static_cast<size_t>(g->B) * 4);
  g->o_ccnt = g->o_hist + static_cast<size_t>(g->B) * kTopkBins * 4;
  g->cand_cap = std::min(kCandCap, static_cast<int>(round_up(std::max(g->max_nc, 64), 64)));
  g->o_cand = cv.take(static_cast<size_t>(g->B) * g->cand_cap * 8);
  g->o_rinfo = cv.take(static_cast<size_t>(g->B) * 4 * 4);   // threshold bin, above, in bin
  g->total = cv.off;
  return QSA_OK;
}

}  // namespace

// =====================================================================================
extern "C" {

const char* qsa_status_string(qsa_status s) {
  switch (s) {
    case QSA_OK: return "QSA_OK";
    case QSA_ERR_INVALID_ARG: return "QSA_ERR_INVALID_ARG";
    case QSA_ERR_ALIGNMENT: return "QSA_ERR_ALIGNMENT";
    case QSA_ERR_CAPACITY: return "QSA_ERR_CAPACITY";
    case QSA_ERR_WORKSPACE: return "QSA_ERR_WORKSPACE";
    case QSA_ERR_CUDA: return "QSA_ERR_CUDA";
    case QSA_ERR_TIMEOUT: return "QSA_ERR_TIMEOUT";
    case QSA_ERR_DEVICE: return "QSA_ERR_DEVICE";
    case QSA_ERR_UNSUPPORTED: return "QSA_ERR_UNSUPPORTED";
  }
  return "QSA_ERR_UNKNOWN";
}

int32_t qsa_version(void) { return kVersion; }

uint64_t qsa_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

qsa_status qsa_workspace_init(void* workspace, size_t ws_bytes, qsa_stream_t stream) {
  if (!workspace) return QSA_ERR_INVALID_ARG;
  if (ws_bytes < QSA_WS_HEADER_BYTES) return QSA_ERR_WORKSPACE;
  if (cudaMemsetAsync(workspace, 0, QSA_WS_HEADER_BYTES, reinterpret_cast<cudaStream_t>(stream)) !=
      cudaSuccess)
    return QSA_ERR_CUDA;
  return QSA_OK;
}

qsa_status qsa_last_device_error(void* workspace, qsa_stream_t stream, uint32_t* site) {
  if (!workspace) return QSA_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint32_t h[4] = {0, 0, 0, 0};
  if (cudaMemcpyAsync(h, workspace, sizeof(h), cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return QSA_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return QSA_ERR_CUDA;
  if (h[0] != 0) {
    if (cudaMemsetAsync(workspace, 0, 16, s) != cudaSuccess) return QSA_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return QSA_ERR_CUDA;
  }
  if (site) *site = h[1];
  if (h[0] == 0) return QSA_OK;
  return h[0] == kErrTimeout ? QSA_ERR_TIMEOUT : QSA_ERR_DEVICE;
}

// ---- step a1 -------------------------------------------------------------------------
size_t qsa_compress_workspace_size(int32_t num_seqs) {
  if (num_seqs <= 0) return 0;
  Carver c;
  c.take(sizeof(SeqMeta) * (num_seqs + 1));
  return c.off;
}

qsa_status qsa_compress(const void* k_idx, const int32_t* d_cu_seqlens, const int32_t* h_cu_seqlens,
                        int32_t num_seqs, void* kbar, void* workspace, size_t ws_bytes,
                        qsa_stream_t stream) {
  qsa_status st = check_prefill_ptrs({k_idx, d_cu_seqlens, kbar, workspace});
  if (st != QSA_OK) return st;
  qsa_params p{512, 1, 0, 0};
  PrefillGeom g;
  st = prefill_geom(h_cu_seqlens, num_seqs, p, &g);
  if (st != QSA_OK) return st;
  if (ws_bytes < qsa_compress_workspace_size(num_seqs)) return QSA_ERR_WORKSPACE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  unsigned char* ws = reinterpret_cast<unsigned char*>(workspace);
  SeqMeta* meta = reinterpret_cast<SeqMeta*>(ws + QSA_WS_HEADER_BYTES);
  st = launch_meta(d_cu_seqlens, num_seqs, 1, meta, dev_status(ws), s);
  if (st != QSA_OK) return st;
  return launch_compress(k_idx, meta, num_seqs, g.total_blocks, kbar, s);
}

// ---- step a2 alone -----------------------------------------------------------------------
qsa_status qsa_index_scores(const void* q_idx, const void* w, const void* kbar,
                            const int32_t* d_cu_seqlens, const int32_t* h_cu_seqlens,
                            int32_t num_seqs, int64_t row_begin, int64_t row_end, float* scores,
                            int64_t ld, int32_t topk, void* workspace, size_t ws_bytes,
                            qsa_stream_t stream) {
  qsa_status st = check_prefill_ptrs({q_idx, w, kbar, d_cu_seqlens, scores, workspace});
  if (st != QSA_OK) return st;
  qsa_params p{topk > 0 ? topk : 512, 1, 0, 0};
  PrefillGeom g;
  st = prefill_geom(h_cu_seqlens, num_seqs, p, &g);
  if (st != QSA_OK) return st;
  if (ws_bytes < g.total) return QSA_ERR_WORKSPACE;
  if (ld < std::max<int64_t>(g.max_nc, 1) || ld % 4 != 0) return QSA_ERR_INVALID_ARG;
  if (row_begin < 0 || row_end > g.T || row_begin >= row_end) return QSA_ERR_INVALID_ARG;
  std::vector<int64_t> starts;
  score_tile_token_starts(h_cu_seqlens, num_seqs, &starts);
  const auto tb = std::lower_bound(starts.begin(), starts.end(), row_begin);
  const auto te = std::lower_bound(starts.begin(), starts.end(), row_end);
  if (tb == starts.end() || *tb != row_begin || te == starts.end() || *te != row_end)
    return QSA_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  unsigned char* ws = reinterpret_cast<unsigned char*>(workspace);
  SeqMeta* meta = reinterpret_cast<SeqMeta*>(ws + g.o_meta);
  st = launch_meta(d_cu_seqlens, num_seqs, g.R, meta, dev_status(ws), s);
  if (st != QSA_OK) return st;
  CUtensorMap tm_kbar, tm_qidx;
  {
    const uint64_t dims[2] = {64, static_cast<uint64_t>(std::max<int64_t>(g.total_blocks, 1))};
    const uint64_t strides[1] = {128};
    const uint32_t box[2] = {64, 128};
    if (!make_tmap(&tm_kbar, kbar, 2, dims, strides, box)) return QSA_ERR_CUDA;
  }
  {
    const uint64_t dims[2] = {64, static_cast<uint64_t>(g.T) * 16};
    const uint64_t strides[1] = {128};
    const uint32_t box[2] = {64, 256};
    if (!make_tmap(&tm_qidx, q_idx, 2, dims, strides, box)) return QSA_ERR_CUDA;
  }
  using C = ScoreCfg<16>;
  const int smem = std::max(C::kSmemBytes, 116 * 1024);
  if (!set_smem(k_index_score<16>, smem)) return QSA_ERR_CUDA;
  ScoreArgs a{};
  a.meta = meta;
  a.num_seqs = num_seqs;
  a.tile_begin = static_cast<int32_t>(tb - starts.begin());
  a.tile_count = static_cast<int32_t>(te - tb);
  a.topk_skip = topk > 0 ? topk : 0;
  a.row_begin = row_begin;
  a.w = reinterpret_cast<const __nv_bfloat16*>(w);
  a.scores = scores;
  a.ld = ld;
  a.st = dev_status(ws);
  k_index_score<16><<<a.tile_count, C::kThreads, smem, s>>>(tm_kbar, tm_qidx, a);
  QSA_CHECK_LAUNCH();
  return QSA_OK;
}

// ---- step a3 alone -----------------------------------------------------------------------
qsa_status qsa_topk(const float* scores, int64_t ld, const int32_t* n_c, int64_t rows, int32_t topk,
                    int32_t max_n_c, int32_t* idx, int32_t* cnt, qsa_stream_t stream) {
  qsa_status st = check_prefill_ptrs({scores, n_c, idx, cnt});
  if (st != QSA_OK) return st;
  if (rows <= 0 || topk < 1 || topk > QSA_MAX_TOPK || max_n_c < 0 || ld < std::max(max_n_c, 1))
    return QSA_ERR_INVALID_ARG;
  return launch_topk(scores, ld, n_c, rows, topk, max_n_c, idx, cnt,
                     reinterpret_cast<cudaStream_t>(stream));
}

// ---- prefill -----------------------------------------------------------------------------
size_t qsa_prefill_workspace_size(const int32_t* h_cu_seqlens, int32_t num_seqs, qsa_params params) {
  PrefillGeom g;
  if (prefill_geom(h_cu_seqlens, num_seqs, params, &g) != QSA_OK) return 0;
  return g.total;
}

static qsa_status prefill_common(const void* q, const void* k, const void* v, const void* q_idx,
                                 const void* k_idx, const void* w, const int32_t* d_cu,
                                 const int32_t* h_cu, int32_t num_seqs, void* out, int32_t* idx_ext,
                                 int32_t* cnt_ext, const int32_t* idx_in, const int32_t* cnt_in,
                                 void* workspace, size_t ws_bytes, qsa_params params,
                                 qsa_stream_t stream) {
  PrefillGeom g;
  qsa_status st = prefill_geom(h_cu, num_seqs, params, &g);
  if (st != QSA_OK) return st;
  if (ws_bytes < g.total) return QSA_ERR_WORKSPACE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  unsigned char* ws = reinterpret_cast<unsigned char*>(workspace);
  SeqMeta* meta = reinterpret_cast<SeqMeta*>(ws + g.o_meta);
  st = launch_meta(d_cu, num_seqs, g.R, meta, dev_status(ws), s);
  if (st != QSA_OK) return st;
  const int32_t* idx_use = idx_in;
  const int32_t* cnt_use = cnt_in;
  if (!idx_in) {
    int32_t* idx = idx_ext ? idx_ext : reinterpret_cast<int32_t*>(ws + g.o_idx);
    int32_t* cnt = cnt_ext ? cnt_ext : reinterpret_cast<int32_t*>(ws + g.o_cnt);
    void* kbar = ws + g.o_kbar;
    st = launch_compress(k_idx, meta, num_seqs, g.total_blocks, kbar, s);
    if (st != QSA_OK) return st;
    {
      const int64_t threads = 256;
      const int grid = static_cast<int>(std::min<int64_t>((g.T + threads - 1) / threads,
                                                          int64_t(num_sms()) * 8));
      k_row_nc<<<grid, threads, 0, s>>>(meta, num_seqs, g.T, reinterpret_cast<int32_t*>(ws + g.o_nc));
      QSA_CHECK_LAUNCH();
    }
    st = run_scores_and_topk(q_idx, w, kbar, h_cu, num_seqs, g, ws, idx, cnt, s);
    if (st != QSA_OK) return st;
    idx_use = idx;
    cnt_use = cnt;
  }
  if (out) return run_attention(q, k, v, idx_use, cnt_use, num_seqs, g, ws, out, s);
  return QSA_OK;
}

qsa_status qsa_prefill(const void* q, const void* k, const void* v, const void* q_idx,
                       const void* k_idx, const void* w, const int32_t* d_cu_seqlens,
                       const int32_t* h_cu_seqlens, int32_t num_seqs, void* out, void* workspace,
                       size_t ws_bytes, qsa_params params, qsa_stream_t stream) {
  qsa_status st = check_prefill_ptrs({q, k, v, q_idx, k_idx, w, d_cu_seqlens, out, workspace});
  if (st != QSA_OK) return st;
  return prefill_common(q, k, v, q_idx, k_idx, w, d_cu_seqlens, h_cu_seqlens, num_seqs, out,
                        nullptr, nullptr, nullptr, nullptr, workspace, ws_bytes, params, stream);
}

qsa_status qsa_prefill_select(const void* q_idx, const void* k_idx, const void* w,
                              const int32_t* d_cu_seqlens, const int32_t* h_cu_seqlens,
                              int32_t num_seqs, int32_t* idx, int32_t* cnt, void* workspace,
                              size_t ws_bytes, qsa_params params, qsa_stream_t stream) {
  qsa_status st = check_prefill_ptrs({q_idx, k_idx, w, d_cu_seqlens, idx, cnt, workspace});
  if (st != QSA_OK) return st;
  return prefill_common(nullptr, nullptr, nullptr, q_idx, k_idx, w, d_cu_seqlens, h_cu_seqlens,
                        num_seqs, nullptr, idx, cnt, nullptr, nullptr, workspace, ws_bytes, params,
                        stream);
}

qsa_status qsa_sparse_attention(const void* q, const void* k, const void* v, const int32_t* idx,
                                const int32_t* cnt, const int32_t* d_cu_seqlens,
                                const int32_t* h_cu_seqlens, int32_t num_seqs, void* out,
                                void* workspace, size_t ws_bytes, qsa_params params,
                                qsa_stream_t stream) {
  qsa_status st = check_prefill_ptrs({q, k, v, idx, cnt, d_cu_seqlens, out, workspace});
  if (st != QSA_OK) return st;
  return prefill_common(q, k, v, nullptr, nullptr, nullptr, d_cu_seqlens, h_cu_seqlens, num_seqs,
                        out, nullptr, nullptr, idx, cnt, workspace, ws_bytes, params, stream);
}

// ---- append ------------------------------------------------------------------------------
}  // extern "C"

namespace {
qsa_status append_impl(const CacheView& view, const void* k, const void* v, const void* k_idx,
                       int32_t n_new, const int32_t* counts, const int32_t* h_len,
                       qsa_stream_t stream) {
  const qsa_cache* cache = view.c;
  if (!cache || !h_len) return QSA_ERR_INVALID_ARG;
  qsa_status st = check_prefill_ptrs({k, v, k_idx, cache->k_blocks, cache->v_blocks, cache->kbar,
                                      cache->kbar_partial, cache->len});
  if (st != QSA_OK) return st;
  if (counts && !aligned16(counts)) return QSA_ERR_ALIGNMENT;
  if (cache->batch <= 0 || cache->capacity <= 0 || cache->capacity % 4 != 0 ||
      cache->capacity > QSA_MAX_SEQ_LEN || n_new < 0)
    return QSA_ERR_INVALID_ARG;
  if (n_new == 0) return QSA_OK;
  for (int b = 0; b < cache->batch; ++b) {
    if (h_len[b] < 0 || h_len[b] > cache->capacity) return QSA_ERR_INVALID_ARG;
    if (!counts && static_cast<int64_t>(h_len[b]) + n_new > cache->capacity) return QSA_ERR_CAPACITY;
  }
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  AppendParams p{};
  p.k = reinterpret_cast<const uint4*>(k);
  p.v = reinterpret_cast<const uint4*>(v);
  p.k_idx = reinterpret_cast<const uint4*>(k_idx);
  p.counts = counts;
  p.n_new = n_new;
  p.batch = cache->batch;
  p.capacity = cache->capacity;
  p.k_blocks = reinterpret_cast<uint4*>(cache->k_blocks);
  p.v_blocks = reinterpret_cast<uint4*>(cache->v_blocks);
  p.kbar = reinterpret_cast<uint4*>(cache->kbar);
  p.partial = cache->kbar_partial;
  p.len = cache->len;
  p.pg = view.pg;
  p.st = DevStatus{nullptr};
  const int sms = num_sms();
  {
    const int slots = (n_new + 3) / 4 + 1;   // blocks a sequence's new tokens can touch
    const int64_t n = static_cast<int64_t>(p.batch) * n_new * 32 + static_cast<int64_t>(p.batch) * slots * 8;
    const int grid = static_cast<int>(std::min<int64_t>((n + 255) / 256, int64_t(sms) * 16));
    QSA_CHECK_PDL(launch_pdl(k_append, dim3(grid), dim3(256), 0, s, p, slots));
  }
  QSA_CHECK_PDL(launch_pdl(k_append_len, dim3((p.batch + 255) / 256), dim3(256), 0, s, cache->len,
                           counts, n_new, p.batch));
  return QSA_OK;
}
}  // namespace

extern "C" {

qsa_status qsa_append_kv(const qsa_cache* cache, const void* k, const void* v, const void* k_idx,
                         int32_t n_new, const int32_t* counts, const int32_t* h_len,
                         qsa_stream_t stream) {
  if (!cache) return QSA_ERR_INVALID_ARG;
  return append_impl(contiguous_view(cache), k, v, k_idx, n_new, counts, h_len, stream);
}

qsa_status qsa_append_kv_paged(const qsa_paged_cache* cache, const void* k, const void* v,
                               const void* k_idx, int32_t n_new, const int32_t* counts,
                               const int32_t* h_len, qsa_stream_t stream) {
  CacheView view;
  const qsa_status st = paged_view(cache, &view);
  if (st != QSA_OK) return st;
  return append_impl(view, k, v, k_idx, n_new, counts, h_len, stream);
}

// ---- decode --------------------------------------------------------------------------------
size_t qsa_decode_workspace_size(const qsa_cache* cache, qsa_params params) {
  DecodeGeom g;
  if (decode_geom(cache, params, &g) != QSA_OK) return 0;
  return g.total;
}

size_t qsa_decode_paged_workspace_size(const qsa_paged_cache* cache, qsa_params params) {
  CacheView view;
  if (paged_view(cache, &view) != QSA_OK) return 0;
  return qsa_decode_workspace_size(&cache->base, params);
}
}  // extern "C"

namespace {
// Decode attention (a6) over the one-token plan records in `plan`: the output directly (one
// split, partials false) or the split partials (m, l, o).
qsa_status launch_decode_attention(const void* q, const CacheView& view, const DecodeGeom& g,
                                   const int32_t* plan, DevStatus dst, void* out, int splits,
                                   float* part_o, float* part_m, float* part_l, bool partials,
                                   cudaStream_t s) {
  const qsa_cache* cache = view.c;
  AttnMaps maps;
  const uint64_t dq[3] = {128, 24, static_cast<uint64_t>(g.B)};
  const uint64_t sq[2] = {256, 24 * 256};
  const uint32_t bq[3] = {64, 12, 1};
  if (!make_tmap(&maps.q, q, 3, dq, sq, bq)) return QSA_ERR_CUDA;
  const uint64_t dkv[2] = {128, static_cast<uint64_t>(view.kv_rows)};
  const uint64_t skv[1] = {256};
  for (int j = 0; j < kNumBoxSizes; ++j) {
    const uint32_t bkv[2] = {64, 4u << j};
    if (!make_tmap(&maps.k[j], cache->k_blocks, 2, dkv, skv, bkv)) return QSA_ERR_CUDA;
    if (!make_tmap(&maps.v[j], cache->v_blocks, 2, dkv, skv, bkv)) return QSA_ERR_CUDA;
  }
  const qsa_status pst = prepare_attention();
  if (pst != QSA_OK) return pst;
  if (view.kv_rows >= 0x7fffffffll) return QSA_ERR_UNSUPPORTED;
  AttnArgs a{};
  a.oob_row = static_cast<int32_t>(view.kv_rows);
  a.pg = view.pg;
  a.plan = plan;
  a.pl = g.pl;
  a.decode = 1;
  a.splits = splits;
  a.cap_blocks = g.cap / 4;
  a.part_o = part_o;
  a.part_m = part_m;
  a.part_l = part_l;
  a.st = dst;
  a.fault_tile = -1;
  a.partials = partials ? 1 : 0;
  a.out = reinterpret_cast<__nv_bfloat16*>(out);   // written directly with one split
  dim3 grid(g.B, 2, splits);
  if (view.pg.table != nullptr) {
    QSA_CHECK_PDL(launch_pdl(k_sparse_attn<true, true>, grid, dim3(AttnCfg::kThreads),
                             AttnCfg::kSmemBytes, s, maps, a));
  } else {
    QSA_CHECK_PDL(launch_pdl(k_sparse_attn<true>, grid, dim3(AttnCfg::kThreads),
                             AttnCfg::kSmemBytes, s, maps, a));
  }
  return QSA_OK;
}

// One shard of a context split over several caches (context-sharded decode).
struct ShardOpt {
  const int32_t* glen = nullptr;   // device [B]: the sequences' whole lengths
  int32_t block0 = 0;              // global block of the shard's first block
  float* cand_score = nullptr;     // selection only: scores of the proposed blocks
};

qsa_status decode_impl(const void* q, const CacheView& view, const void* q_idx, const void* w,
                       void* out, const int32_t* h_len, int32_t* sel_idx, int32_t* sel_cnt,
                       void* workspace, size_t ws_bytes, qsa_params params, qsa_stream_t stream,
                       const ShardOpt* shard = nullptr) {
  const qsa_cache* cache = view.c;
  if (!cache || !h_len) return QSA_ERR_INVALID_ARG;
  qsa_status st = shard ? check_prefill_ptrs({q_idx, w, workspace, cache->kbar, cache->len,
                                              shard->glen, shard->cand_score, sel_idx, sel_cnt})
                        : check_prefill_ptrs({q, q_idx, w, out, workspace, cache->k_blocks,
                                              cache->v_blocks, cache->kbar, cache->len});
  if (st != QSA_OK) return st;
  if (shard && (shard->block0 < 0 || shard->block0 % 128 != 0)) return QSA_ERR_INVALID_ARG;
  if ((sel_idx && !aligned16(sel_idx)) || (sel_cnt && !aligned16(sel_cnt))) return QSA_ERR_ALIGNMENT;
  DecodeGeom g;
  st = decode_geom(cache, params, &g);
  if (st != QSA_OK) return st;
  if (ws_bytes < g.total) return QSA_ERR_WORKSPACE;
  int max_len = 0;
  for (int b = 0; b < g.B; ++b) {
    if (h_len[b] < (shard ? 0 : 1) || h_len[b] > g.cap) return QSA_ERR_INVALID_ARG;
    max_len = std::max(max_len, h_len[b]);
  }
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  unsigned char* ws = reinterpret_cast<unsigned char*>(workspace);
  float* scores = reinterpret_cast<float*>(ws + g.o_scores);
  int32_t* n_c = reinterpret_cast<int32_t*>(ws + g.o_nc);
  int32_t* idx = sel_idx ? sel_idx : reinterpret_cast<int32_t*>(ws + g.o_idx);
  int32_t* cnt = sel_cnt ? sel_cnt : reinterpret_cast<int32_t*>(ws + g.o_cnt);
  int32_t* plan = reinterpret_cast<int32_t*>(ws + g.o_plan);
  uint32_t* hist = reinterpret_cast<uint32_t*>(ws + g.o_hist);
  int32_t* cand_cnt = reinterpret_cast<int32_t*>(ws + g.o_ccnt);
  uint64_t* cand = reinterpret_cast<uint64_t*>(ws + g.o_cand);
  int32_t* rinfo = reinterpret_cast<int32_t*>(ws + g.o_rinfo);
  const int sms = num_sms();
  // candidate blocks of the longest row: those before the query's own block, or for a shard
  // at most every complete block it holds
  const int max_nc_now = shard ? max_len / 4 : (max_len - 1) / 4;
  // the decode kernels form one chain of programmatic dependent launches (each waits for the
  // one before it); the first also follows the caller's last kernel (the append) that way
  {
    const int64_t words = static_cast<int64_t>(g.B) * (kTopkBins + 1);
    const int grid = static_cast<int>(std::min<int64_t>((words + 255) / 256, int64_t(sms) * 4));
    QSA_CHECK_PDL(launch_pdl(k_zero_words, dim3(grid), dim3(256), 0, s, hist, words));
  }
  // a2: scores, with the first radix digit's histogram of every row (one token x 16 heads per sequence, split over M-tiles)
  {
    CUtensorMap tm_kbar, tm_qidx;
    const uint64_t dk[2] = {64, static_cast<uint64_t>(view.kbar_rows)};
    const uint64_t sk[1] = {128};
    const uint32_t bk[2] = {64, 128};
    if (!make_tmap(&tm_kbar, cache->kbar, 2, dk, sk, bk)) return QSA_ERR_CUDA;
    const uint64_t dq[2] = {64, static_cast<uint64_t>(g.B) * 16};
    const uint32_t bq[2] = {64, 16};
    if (!make_tmap(&tm_qidx, q_idx, 2, dq, sk, bq)) return QSA_ERR_CUDA;
    using C = ScoreCfg<1>;
    if (!set_smem(k_index_score<1>, C::kSmemBytes)) return QSA_ERR_CUDA;
    // split each sequence's M-tiles over CTAs: fewest waves x tiles per CTA over the SMs'
    // CTA slots, counting a fixed cost of two tiles per CTA for its setup and histogram flush
    const int total_mt = std::max(1, (max_nc_now + 127) / 128);
    const int64_t slots = int64_t(sms) * C::kCtasPerSm;
    int splits = 1, per = total_mt;
    int64_t best = -1;
    for (int sp = 1; sp <= std::min(total_mt, 256); ++sp) {
      const int pr = (total_mt + sp - 1) / sp;
      const int se = (total_mt + pr - 1) / pr;
      const int64_t waves = (int64_t(g.B) * se + slots - 1) / slots;
      const int64_t cost = waves * (pr + 2);
      if (best < 0 || cost < best) {
        best = cost;
        splits = se;
        per = pr;
      }
    }
    ScoreArgs a{};
    a.len = cache->len;
    a.splits = splits;
    a.mtiles_per_split = per;
    a.kbar_rows_per_seq = g.cap / 4;
    a.pg = view.pg;
    a.kbar_oob_row = static_cast<int32_t>(view.kbar_rows);
    a.n_c_out = n_c;
    a.hist = hist;
    if (shard) {
      a.glen = shard->glen;
      a.block0 = shard->block0;
    }
    a.w = reinterpret_cast<const __nv_bfloat16*>(w);
    a.scores = scores;
    a.ld = g.ld;
    a.st = dev_status(ws);
    QSA_CHECK_PDL(launch_pdl(k_index_score<1>, dim3(g.B * splits), dim3(C::kThreads),
                             C::kSmemBytes, s, tm_kbar, tm_qidx, a));
  }
  // a3: top-k: candidates at or above the threshold bin, then the exact select per row
  {
    // up to one pass of kCollectPerCta scores per CTA, and no more CTAs than one wave (one
    // CTA of 512 threads per SM)
    const int parts = std::max(1, std::min((max_nc_now + kCollectPerCta - 1) / kCollectPerCta,
                                           sms / g.B));
    QSA_CHECK_PDL(launch_pdl(k_topk_collect, dim3(g.B * parts), dim3(kCandThreads), 0, s,
                             static_cast<const float*>(scores), g.ld,
                             static_cast<const int32_t*>(n_c), g.topk, parts, g.cand_cap,
                             static_cast<const uint32_t*>(hist), cand_cnt, cand, rinfo));
    const int smem = g.finish_smem();
    if (!set_smem(k_topk_finish, smem)) return QSA_ERR_CUDA;
    // also writes each sequence's attention plan record
    QSA_CHECK_PDL(launch_pdl(k_topk_finish, dim3(g.B), dim3(kTopkThreads), smem, s,
                             static_cast<const float*>(scores), g.ld,
                             static_cast<const int32_t*>(n_c), g.topk, g.cand_cap,
                             std::max(g.max_nc, 1), static_cast<const uint32_t*>(hist),
                             static_cast<const int32_t*>(cand_cnt),
                             static_cast<const uint64_t*>(cand),
                             static_cast<const int32_t*>(rinfo), idx, cnt,
                             static_cast<const int32_t*>(cache->len), g.pl,
                             shard ? nullptr : plan, shard ? shard->cand_score : nullptr,
                             shard ? shard->block0 : 0));
  }
  if (shard) return QSA_OK;   // a shard's selection stops at its candidates
  // a6: split attention + combine
  {
    float* part_o = reinterpret_cast<float*>(ws + g.o_po);
    float* part_m = reinterpret_cast<float*>(ws + g.o_pm);
    float* part_l = reinterpret_cast<float*>(ws + g.o_pl);
    st = launch_decode_attention(q, view, g, plan, dev_status(ws), out, g.splits, part_o, part_m,
                                 part_l, false, s);
    if (st != QSA_OK) return st;
    if (g.splits > 1) {
      const int warps = g.B * kHeads;
      QSA_CHECK_PDL(launch_pdl(k_decode_combine, dim3((warps * 32 + 255) / 256), dim3(256), 0, s,
                               static_cast<const float*>(part_o),
                               static_cast<const float*>(part_m),
                               static_cast<const float*>(part_l), g.B, g.splits,
                               reinterpret_cast<__nv_bfloat16*>(out)));
    }
  }
  return QSA_OK;
}
}  // namespace

extern "C" {

qsa_status qsa_decode(const void* q, const qsa_cache* cache, const void* q_idx, const void* w,
                      void* out, const int32_t* h_len, int32_t* sel_idx, int32_t* sel_cnt,
                      void* workspace, size_t ws_bytes, qsa_params params, qsa_stream_t stream) {
  if (!cache) return QSA_ERR_INVALID_ARG;
  return decode_impl(q, contiguous_view(cache), q_idx, w, out, h_len, sel_idx, sel_cnt, workspace,
                     ws_bytes, params, stream);
}

qsa_status qsa_decode_paged(const void* q, const qsa_paged_cache* cache, const void* q_idx,
                            const void* w, void* out, const int32_t* h_len, int32_t* sel_idx,
                            int32_t* sel_cnt, void* workspace, size_t ws_bytes, qsa_params params,
                            qsa_stream_t stream) {
  CacheView view;
  const qsa_status st = paged_view(cache, &view);
  if (st != QSA_OK) return st;
  return decode_impl(q, view, q_idx, w, out, h_len, sel_idx, sel_cnt, workspace, ws_bytes, params,
                     stream);
}

// ---- context-sharded decode ---------------------------------------------------------------
size_t qsa_decode_shard_workspace_size(const qsa_cache* shard, qsa_params params) {
  return qsa_decode_workspace_size(shard, params);
}

qsa_status qsa_decode_shard_select(const void* q_idx, const void* w, const qsa_cache* shard,
                                   int32_t block0, const int32_t* d_glen, const int32_t* h_len,
                                   float* cand_score, int32_t* cand_idx, int32_t* cand_cnt,
                                   void* workspace, size_t ws_bytes, qsa_params params,
                                   qsa_stream_t stream) {
  if (!shard) return QSA_ERR_INVALID_ARG;
  ShardOpt o;
  o.glen = d_glen;
  o.block0 = block0;
  o.cand_score = cand_score;
  return decode_impl(nullptr, contiguous_view(shard), q_idx, w, nullptr, h_len, cand_idx,
                     cand_cnt, workspace, ws_bytes, params, stream, &o);
}

qsa_status qsa_merge_candidates(const float* cand_score, const int32_t* cand_idx,
                                const int32_t* cand_cnt, int32_t shards, int32_t batch,
                                int32_t topk, int32_t max_blocks, int32_t* sel_idx,
                                int32_t* sel_cnt, void* workspace, size_t ws_bytes,
                                qsa_stream_t stream) {
  qsa_status st = check_prefill_ptrs({cand_score, cand_idx, cand_cnt, sel_idx, sel_cnt, workspace});
  if (st != QSA_OK) return st;
  if (shards < 1 || shards > kMaxShards || batch < 1 || topk < 1 || topk > QSA_MAX_TOPK ||
      max_blocks < 1 || max_blocks > QSA_MAX_SEQ_LEN / 4)
    return QSA_ERR_INVALID_ARG;
  if (ws_bytes < QSA_WS_HEADER_BYTES) return QSA_ERR_WORKSPACE;
  const int nwords = (max_blocks + 31) / 32;
  const int64_t smem = kTopkSharedBytes + int64_t(shards) * topk * 8 + 2 * int64_t(nwords) * 4;
  if (smem > 227 * 1024) return QSA_ERR_UNSUPPORTED;
  if (!set_smem(k_merge_candidates, static_cast<int>(smem))) return QSA_ERR_CUDA;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  QSA_CHECK_PDL(launch_pdl(k_merge_candidates, dim3(batch), dim3(kTopkThreads),
                           static_cast<size_t>(smem), s, cand_score, cand_idx, cand_cnt, shards,
                           batch, topk, nwords, sel_idx, sel_cnt, dev_status(workspace)));
  return QSA_OK;
}

qsa_status qsa_decode_shard_attend(const void* q, const qsa_cache* shard, int32_t block0,
                                   const int32_t* d_glen, const int32_t* sel_idx,
                                   const int32_t* sel_cnt, float* part_o, float* part_m,
                                   float* part_l, void* workspace, size_t ws_bytes,
                                   qsa_params params, qsa_stream_t stream) {
  if (!shard) return QSA_ERR_INVALID_ARG;
  qsa_status st = check_prefill_ptrs({q, shard->k_blocks, shard->v_blocks, d_glen, sel_idx,
                                      sel_cnt, part_o, part_m, part_l, workspace});
  if (st != QSA_OK) return st;
  if (block0 < 0 || block0 % 128 != 0) return QSA_ERR_INVALID_ARG;
  DecodeGeom g;
  st = decode_geom(shard, params, &g);
  if (st != QSA_OK) return st;
  if (ws_bytes < g.total) return QSA_ERR_WORKSPACE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  unsigned char* ws = reinterpret_cast<unsigned char*>(workspace);
  int32_t* plan = reinterpret_cast<int32_t*>(ws + g.o_plan);
  QSA_CHECK_PDL(launch_pdl(k_shard_plan, dim3(g.B), dim3(kPlanThreads), 0, s, sel_idx, sel_cnt,
                           g.topk, d_glen, block0, g.cap / 4, g.pl, plan, dev_status(ws)));
  return launch_decode_attention(q, contiguous_view(shard), g, plan, dev_status(ws), nullptr, 1,
                                 part_o, part_m, part_l, true, s);
}

qsa_status qsa_combine_partials(const float* part_o, const float* part_m, const float* part_l,
                                int32_t shards, int32_t batch, void* out, qsa_stream_t stream) {
  qsa_status st = check_prefill_ptrs({part_o, part_m, part_l, out});
  if (st != QSA_OK) return st;
  if (shards < 1 || batch < 1) return QSA_ERR_INVALID_ARG;
  const int warps = batch * kHeads;
  QSA_CHECK_PDL(launch_pdl(k_combine_shards, dim3((warps * 32 + 255) / 256), dim3(256), 0,
                           reinterpret_cast<cudaStream_t>(stream), part_o, part_m, part_l, batch,
                           shards, reinterpret_cast<__nv_bfloat16*>(out)));
  return QSA_OK;
}

}  // extern "C"

// ---- decode with the library's own fixed scratch -----------------------------------------
// One device array per GPU that loads the library, used as the workspace of
// qsa_decode_noalloc.  In host code its name only stands for the symbol; the device
// address comes from cudaGetSymbolAddress with the device current.
static __device__ __align__(256) unsigned char g_noalloc_scratch[QSA_NOALLOC_SCRATCH_BYTES];

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kMaxDevices] = {};

// The array's address on the current device.  It is looked up again on every call made
// outside a stream capture (so that a module reloaded after cudaDeviceReset is followed);
// during a capture the address of the last uncaptured call on this device is used, since a
// capture must not call into the runtime for the symbol (make one call before capturing).
qsa_status noalloc_scratch(cudaStream_t s, void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return QSA_ERR_CUDA;
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(s, &cs) != cudaSuccess) return QSA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (cs == cudaStreamCaptureStatusNone) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return QSA_ERR_CUDA;
    g_noalloc_ptr[dev] = p;
  } else if (!g_noalloc_ptr[dev]) {
    return QSA_ERR_CUDA;   // no uncaptured call yet on this device
  }
  *out = g_noalloc_ptr[dev];
  return QSA_OK;
}
}  // namespace

extern "C" qsa_status qsa_decode_noalloc(const void* q, const qsa_cache* cache, const void* q_idx,
                                         const void* w, void* out, const int32_t* h_len,
                                         int32_t* sel_idx, int32_t* sel_cnt, qsa_params params,
                                         qsa_stream_t stream) {
  if (!cache) return QSA_ERR_INVALID_ARG;
  const size_t need = qsa_decode_workspace_size(cache, params);
  if (need == 0) return QSA_ERR_INVALID_ARG;
  if (need > QSA_NOALLOC_SCRATCH_BYTES) {
    fprintf(stderr,
            "qsa_decode_noalloc: this cache needs %zu bytes of scratch, more than the fixed "
            "%u bytes; use qsa_decode with a workspace\n",
            need, static_cast<unsigned>(QSA_NOALLOC_SCRATCH_BYTES));
    return QSA_ERR_WORKSPACE;
  }
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  void* ws = nullptr;
  qsa_status st = noalloc_scratch(s, &ws);
  if (st != QSA_OK) return st;
  // the status words must start at zero; everything else is written before it is read
  if (cudaMemsetAsync(ws, 0, QSA_WS_HEADER_BYTES, s) != cudaSuccess) return QSA_ERR_CUDA;
  return qsa_decode(q, cache, q_idx, w, out, h_len, sel_idx, sel_cnt, ws,
                    QSA_NOALLOC_SCRATCH_BYTES, params, stream);
}

extern "C" qsa_status qsa_noalloc_last_device_error(qsa_stream_t stream, uint32_t* site) {
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint32_t h[4] = {0, 0, 0, 0};
  if (cudaMemcpyFromSymbolAsync(h, g_noalloc_scratch, sizeof(h), 0, cudaMemcpyDeviceToHost, s) !=
      cudaSuccess)
    return QSA_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return QSA_ERR_CUDA;
  if (h[0] != 0) {
    static const uint32_t zero[4] = {0, 0, 0, 0};
    if (cudaMemcpyToSymbolAsync(g_noalloc_scratch, zero, sizeof(zero), 0, cudaMemcpyHostToDevice,
                                s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess)
      return QSA_ERR_CUDA;
  }
  if (site) *site = h[1];
  if (h[0] == 0) return QSA_OK;
  return h[0] == kErrTimeout ? QSA_ERR_TIMEOUT : QSA_ERR_DEVICE;
}

// ---- the Gated DeltaNet layer ------------------------------------------------------------
extern "C" qsa_status qsa_gated_deltanet(const void* q, const void* k, const void* v,
                                         const float* log_alpha, const float* beta,
                                         const int32_t* d_cu_seqlens, const int32_t* h_cu_seqlens,
                                         int32_t num_seqs, int32_t heads, void* out,
                                         float* final_state, qsa_stream_t stream) {
  if (!q || !k || !v || !log_alpha || !beta || !d_cu_seqlens || !h_cu_seqlens || !out)
    return QSA_ERR_INVALID_ARG;
  if (num_seqs < 1 || num_seqs > 65535 || heads < 1 || heads > 256) return QSA_ERR_INVALID_ARG;
  if (h_cu_seqlens[0] != 0) return QSA_ERR_INVALID_ARG;
  for (int32_t i = 0; i < num_seqs; ++i)
    if (h_cu_seqlens[i + 1] < h_cu_seqlens[i]) return QSA_ERR_INVALID_ARG;
  for (const void* p : {q, k, v, static_cast<const void*>(out)})
    if (!aligned16(p)) return QSA_ERR_ALIGNMENT;
  if (!set_smem(k_gated_deltanet, kGdnSmemBytes)) return QSA_ERR_CUDA;
  GdnArgs a{};
  a.q = static_cast<const __nv_bfloat16*>(q);
  a.k = static_cast<const __nv_bfloat16*>(k);
  a.v = static_cast<const __nv_bfloat16*>(v);
  a.log_alpha = log_alpha;
  a.beta = beta;
  a.cu = d_cu_seqlens;
  a.heads = heads;
  a.out = static_cast<__nv_bfloat16*>(out);
  a.final_state = final_state;
  k_gated_deltanet<<<dim3(heads, num_seqs), kGdnThreads, kGdnSmemBytes,
                     reinterpret_cast<cudaStream_t>(stream)>>>(a);
  QSA_CHECK_LAUNCH();
  return QSA_OK;
}
