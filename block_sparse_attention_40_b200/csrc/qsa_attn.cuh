// qsa_attn.cuh -- steps a4/a6: attention over the selected blocks plus the own block.
//
// One CTA handles one attention tile (up to R consecutive query tokens of a sequence, R = 1
// in decode) for one KV head g.  Its 128 tensor-core rows are (token, query head of group g)
// pairs: row = 12 * token + head, rows >= 12R are padding.  Keys are the tile's union of
// selected blocks and own blocks (see k_attn_plan), processed 32 blocks = 128 keys per chunk.
//
// Per chunk i (S and P double-buffered in TMEM; K and V in separate shared-memory rings of 3
// and 2 stages, so K of later chunks streams in while earlier chunks are still in P.V):
//   S = Q K^T        tcgen05, A = Q (smem, K-major), B = K chunk (smem, K-major), D in TMEM;
//                    its completion frees the K slot
//   softmax          one thread per row: keys of blocks the row's token did not select get
//                    -inf (a per-block bias), and so do the own block's future tokens; online
//                    max in the log2 domain with lazy rescaling of O (only when the max grows
//                    by more than 2^8); P = exp2(.) as bf16 into its own TMEM columns, except
//                    for pairs of blocks that no row of the warp attends, whose P is zero
//   O += P V         tcgen05, A = P (TMEM), B = V chunk (smem, MN-major), D = O in TMEM;
//                    its completion frees the V slot
// Decode (kDec, one query token, 12 valid rows): the 12 head rows are loaded into each of the
// four TMEM lane quarters, and each copy takes a quarter of every chunk's keys with its own
// running max and sum, so that all softmax warps share the work instead of one warp per group;
// P then lives in its own TMEM columns and the four copies are merged at the end.
//
// K/V rows are gathered with TMA boxes of 4..128 rows x 64 dims, one per naturally aligned
// power-of-two piece of each run of consecutive blocks (no multicast).  The boxes of a chunk
// are spread over several producer warps (3 for K, 4 for V): on this part the rate at which a
// warp's TMA copies go out is what limits a gather of small boxes, and it adds up over warps.
//
// Warp roles (kSoftGroups = 2: 512 threads): warps 0-7 softmax (warp w owns TMEM lanes
// 32(w%4)..+31; warpgroup g handles keys 64g..64g+63 of each chunk), warp 8 TMEM allocation +
// MMA issue, warps 9-11 K producers (warp 9 also loads Q), warps 12-15 V producers.  The
// softmax warpgroups raise their register budget to kRegsSoftmax, the other two lower theirs
// to kRegsOther (setmaxnreg); the host checks before the first launch that the launch's
// registers cover both.  Four softmax warpgroups (32 keys each, 768 threads) measured slower.
#pragma once

#include "qsa_common.cuh"
#include "qsa_misc.cuh"

namespace qsa {

#ifndef QSA_ATTN_SOFT_GROUPS
#define QSA_ATTN_SOFT_GROUPS 2
#endif
struct AttnCfg {
  static constexpr int kSoftGroups = QSA_ATTN_SOFT_GROUPS;   // softmax warpgroups (2 or 4)
  static constexpr int kSoftWarps = 4 * kSoftGroups;
  static constexpr int kMmaWarp = kSoftWarps;
  static constexpr int kKWarp0 = kSoftWarps + 1, kKWarps = 3;
  static constexpr int kVWarp0 = kSoftWarps + 4, kVWarps = 4;
  static constexpr int kThreads = 32 * (kSoftWarps + 8);   // + MMA, 3 K and 4 V producers
  static constexpr int kRegsSoftmax = kSoftGroups == 2 ? 168 : 96;
  static constexpr int kRegsOther = kSoftGroups == 2 ? 80 : 48;
  // registers the launch must provide for the two budgets above (checked on the host)
  static constexpr int kRegsNeeded = 128 * kSoftGroups * kRegsSoftmax + 256 * kRegsOther;
  static constexpr int kChunkBlocks = 32;
  static constexpr int kChunkKeys = 128;
  static constexpr int kQBytes = 128 * kHeadDim * 2;         // 32 KB (2 panels of 16 KB)
  static constexpr int kKVBytes = kChunkKeys * kHeadDim * 2; // 32 KB per K or V chunk
  static constexpr int kKStages = 3;
  static constexpr int kVStages = 2;
  static constexpr int kQOff = 0;
  static constexpr int kKOff = kQBytes;
  static constexpr int kVOff = kKOff + kKStages * kKVBytes;
  static constexpr int kXOff = kVOff + kVStages * kKVBytes;    // row-max / row-sum exchange
  static constexpr int kXBytes = (2 * kSoftGroups * 128 + kSoftGroups * 128) * 4;
  static constexpr int kBarOff = kXOff + kXBytes;
  static constexpr int kNumBars = 1 + 2 * kKStages + 2 * kVStages + 2 + 2 + 2 + 1 + 1 + 1;
  // the block-mask bias table: entry n holds, for bits 0..3 of n, 0 (block selected) or -inf
  static constexpr int kLutOff = (kBarOff + kNumBars * 8 + 16 + 15) / 16 * 16;   // 16 x float4
  static constexpr int kSmemBytes = kLutOff + 256 + 1024;
  static constexpr int kTmemCols = 512;   // S0 [0,128) S1 [128,256) O [256,384)
  static constexpr uint32_t kIdescQK = idesc_bf16_f32(128, 128, 0, 0);
  static constexpr uint32_t kIdescPV = idesc_bf16_f32(128, 128, 0, 1);   // B = V is MN-major
};
static_assert(AttnCfg::kSmemBytes <= 232448, "attention tile exceeds shared memory");

// Tensor maps of one attention launch.  K and V each have six maps whose boxes are 64 dims
// wide and 4, 8, 16, 32, 64, 128 rows high (1..32 consecutive blocks), so that a run of
// consecutive selected blocks is gathered with a few large boxes instead of one per block.
constexpr int kNumBoxSizes = 6;
struct AttnMaps {
  CUtensorMap q;
  CUtensorMap k[kNumBoxSizes];
  CUtensorMap v[kNumBoxSizes];
};

struct AttnArgs {
  const int32_t* plan;     // tile records (PlanLayout)
  int32_t oob_row;         // a K/V row index past the end of the tensor (zero-filled by TMA)
  PlanLayout pl;
  const SeqMeta* meta;     // prefill
  int32_t num_seqs;
  int32_t decode;          // 1: decode (tile = sequence, KV from the block cache)
  int32_t splits;          // chunk splits per tile (decode), 1 for prefill
  int64_t cap_blocks;      // decode: capacity / 4
  Paging pg;               // decode: where each sequence's K/V blocks live (table null: contiguous)
  __nv_bfloat16* out;      // prefill: [T][24][128]; decode with one split: [B][24][128]
  float* part_o;           // decode: [B][2][splits][12][128]
  float* part_m;           // decode: [B][2][splits][12]
  float* part_l;
  DevStatus st;
  int32_t fault_tile = -1; // testing only (-1: off): see k_sparse_attn
  int32_t partials = 0;    // decode: write the (m, l, o) partials even with one split
};

// Testing only: the wait limit of the faulted tile's MMA warp (1 ms).
constexpr uint64_t kFaultWaitNs = 1000000ull;

__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
  return (static_cast<uint64_t>(__float_as_uint(hi)) << 32) | __float_as_uint(lo);
}
__device__ __forceinline__ float f2_lo(uint64_t v) { return __uint_as_float(static_cast<uint32_t>(v)); }
__device__ __forceinline__ float f2_hi(uint64_t v) { return __uint_as_float(static_cast<uint32_t>(v >> 32)); }
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Producer of one operand stream (K or V) of a tile, run by nw warps (this one is number w).
// Lane u of each warp owns union slot u of the chunk.  Maximal runs of consecutive block ids
// (and the run of padding slots past the end of the union) are cut into power-of-two pieces;
// the first lane of each run issues one TMA box per piece (rows 4*blk.., two 64-dim panels).
// Run r of a chunk (in slot order) goes to warp r mod nw; warp 0 posts the chunk's bytes.
// Padding rows come from an out-of-range coordinate and are zero-filled.  skip_first (testing
// only): nothing is posted or copied for the first chunk, so its full barrier never completes
// and the consumer's bounded wait gives up; that chunk is then not drained.  kPaged (a paged
// decode cache): runs are also cut where a page starts, and each run's rows are looked up in
// the page table of sequence seq (KV head g).  The other instances carry none of that code: the
// prefill gather is limited by how fast these warps issue copies.
template <bool kPaged>
__device__ __forceinline__ void attn_producer(const CUtensorMap* maps, unsigned char* ring,
                                              uint64_t* full, uint64_t* empty, int stages,
                                              const int32_t* uni, int U, int c_begin, int nchunks,
                                              int64_t kv_row_base, int col0, int32_t oob_row,
                                              const Paging& pg, int seq, int g,
                                              int w, int nw, volatile int* abort, DevStatus st,
                                              uint32_t site, bool skip_first) {
  const int lane = threadIdx.x & 31;
  int upos = c_begin * AttnCfg::kChunkBlocks + lane;
  int blk_next = upos < U ? uni[upos] : -1;
  // paged: the pool row of the slot's block, looked up a chunk ahead like the block itself
  // (-1: out-of-range page entry); a piece of a run starts off blocks later in the same page
  auto lookup = [&](int b) -> int64_t {
    if constexpr (kPaged) return b >= 0 ? pool_kv_row(pg, seq, g, b) : 0;
    return 0;
  };
  int64_t prow_next = lookup(blk_next);
  int issued = 0;
  for (int i = 0; i < nchunks; ++i) {
    const int blk = blk_next;           // -1: padding slot
    const int64_t prow = prow_next;
    upos += AttnCfg::kChunkBlocks;
    if (i + 1 < nchunks) {
      blk_next = upos < U ? uni[upos] : -1;
      prow_next = lookup(blk_next);
    }
    const int s = i % stages;
    bool ok = true;
    if (lane == 0) ok = mbar_wait(&empty[s], ((i / stages) & 1) ^ 1, abort, st, site);
    ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
    if (!ok) break;
    const bool skip = skip_first && i == 0;
    if (lane == 0 && w == 0 && !skip) mbar_arrive_expect_tx(&full[s], AttnCfg::kKVBytes);
    __syncwarp();
    const int prev = __shfl_up_sync(0xffffffffu, blk, 1);
    bool start = lane == 0 || (blk < 0) != (prev < 0) || (blk >= 0 && blk != prev + 1);
    if constexpr (kPaged) start = start || (blk >= 0 && blk % pg.page_blocks == 0);
    const unsigned starts = __ballot_sync(0xffffffffu, start);
    // (a box may complete before warp 0 posts the bytes: the phase cannot end while the
    // posting arrival is missing)
    if (!skip && start && __popc(starts & ((1u << lane) - 1u)) % nw == w) {
      const unsigned later = starts & ~((2u << lane) - 1u);   // run starts after this lane
      const int run_end = later ? __ffs(later) - 1 : 32;
      int off = 0;
      while (off < run_end - lane) {
        const int rem = run_end - lane - off;
        const int slot = lane + off;
        // the largest power of two that fits the rest of the run and divides the slot: every
        // box starts in shared memory at a multiple of its own size (>= 512 bytes)
        const int lg_fit = 31 - __clz(rem);
        const int lg_align = slot == 0 ? 5 : __ffs(slot) - 1;
        const int lg = lg_fit < lg_align ? lg_fit : lg_align;
        int32_t row = oob_row;
        if (blk >= 0) {
          if constexpr (kPaged) {
            if (prow < 0) report_error(st, kErrDevice, 205);
            else row = static_cast<int32_t>(prow + static_cast<int64_t>(off) * kBlock);
          } else {
            row = static_cast<int32_t>(kv_row_base + static_cast<int64_t>(blk + off) * kBlock);
          }
        }
        unsigned char* dst = ring + s * AttnCfg::kKVBytes + slot * 512;
        tma_load_2d(dst, &maps[lg], col0, row, &full[s]);
        tma_load_2d(dst + 16384, &maps[lg], col0 + 64, row, &full[s]);
        off += 1 << lg;
      }
    }
    __syncwarp();
    ++issued;
  }
  if (lane == 0 && *abort) {
    int from = issued > stages ? issued - stages : 0;
    if (skip_first && from == 0) from = 1;   // nothing was posted for the skipped chunk
    for (int j = from; j < issued; ++j) mbar_drain(&full[j % stages], (j / stages) & 1);
  }
}

// kDec: decode layout (one query token per tile; see the decode softmax below).  kPaged: the
// decode cache is paged (args.pg).
template <bool kDec, bool kPaged = false>
__global__ void __launch_bounds__(AttnCfg::kThreads, 1)
    k_sparse_attn(const __grid_constant__ AttnMaps maps, AttnArgs args) {
  using C = AttnCfg;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  unsigned char* sQ = smem + C::kQOff;
  unsigned char* sK = smem + C::kKOff;
  unsigned char* sV = smem + C::kVOff;
  float* xmax = reinterpret_cast<float*>(smem + C::kXOff);   // [parity][group][128]
  float* xsum = xmax + 2 * C::kSoftGroups * 128;              // [group][128]
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;
  uint64_t* k_empty = k_full + C::kKStages;
  uint64_t* v_full = k_empty + C::kKStages;
  uint64_t* v_empty = v_full + C::kVStages;
  uint64_t* s_full = v_empty + C::kVStages;
  uint64_t* p_full = s_full + 2;
  uint64_t* p_free = p_full + 2;     // P.V of the buffer's last chunk has completed
  uint64_t* pv_done = p_free + 2;
  uint64_t* mma_done = pv_done + 1;
  uint64_t* o_final = mma_done + 1;  // every P.V of the tile has completed
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(bars + C::kNumBars);
  volatile int* s_abort = reinterpret_cast<volatile int*>(s_tmem + 1);

  pdl_trigger();
  pdl_wait();   // decode: the plan records come from the kernel before
  const int g = blockIdx.y;
  const int split = blockIdx.z;
  const int tile = blockIdx.x;
  const int32_t* rec = args.plan + static_cast<int64_t>(tile) * args.pl.stride;
  const int U = rec[0];
  const int ntok = rec[1];
  const int R = args.pl.R;
  const int nchunks_all = (U + C::kChunkBlocks - 1) / C::kChunkBlocks;
  int c_begin = 0, c_end = nchunks_all;
  if (kDec) {
    const int per = (nchunks_all + args.splits - 1) / args.splits;
    c_begin = split * per;
    c_end = c_begin + per < nchunks_all ? c_begin + per : nchunks_all;
  }
  const int nchunks = c_end > c_begin ? c_end - c_begin : 0;

  // where this tile's tokens live
  int64_t tok_row0 = 0;   // global token row (prefill) / sequence (decode) of token 0
  int pos0 = 0;           // position within the sequence of token 0
  int64_t kv_row_base = 0;
  if (kDec) {
    tok_row0 = tile;
    pos0 = rec[2];   // p = len - 1 of the sequence
    kv_row_base = (static_cast<int64_t>(tile) * 2 + g) * args.cap_blocks * kBlock;
  } else {
    const int s = find_seq_of_tile<true>(args.meta, args.num_seqs, tile);
    const int lt = tile - args.meta[s].attn_tile0;
    pos0 = lt * R;
    tok_row0 = args.meta[s].tok0 + pos0;
    kv_row_base = args.meta[s].tok0;
  }

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // Testing only (args.fault_tile >= 0): in that tile (KV head 0, first split) the K producers
  // post nothing for the first chunk and the MMA warp's waits give up after kFaultWaitNs, so
  // the launch reports QSA_ERR_TIMEOUT (site 23) and every warp unwinds through the abort path.
  const bool fault = args.fault_tile >= 0 && tile == args.fault_tile && g == 0 && split == 0;

  if (nchunks == 0 || ntok == 0) {
    // decode split without keys: write an empty partial
    if (kDec && ntok > 0 && threadIdx.x < kGroup) {
      const int64_t pr = ((static_cast<int64_t>(tile) * 2 + g) * args.splits + split) * kGroup +
                         threadIdx.x;
      args.part_m[pr] = -INFINITY;
      args.part_l[pr] = 0.f;
      for (int d = 0; d < kHeadDim; ++d) args.part_o[pr * kHeadDim + d] = 0.f;
    }
    return;
  }

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < C::kKStages; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&k_empty[i], 1);
    }
    for (int i = 0; i < C::kVStages; ++i) {
      mbar_init(&v_full[i], 1);
      mbar_init(&v_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], C::kSoftWarps);
      mbar_init(&p_free[i], 1);
    }
    mbar_init(pv_done, 1);
    mbar_init(mma_done, 1);
    mbar_init(o_final, 1);
    *s_abort = 0;
    fence_mbar_init();
  }
  if (threadIdx.x < 64)
    reinterpret_cast<float*>(smem + C::kLutOff)[threadIdx.x] =
        (((threadIdx.x >> 2) >> (threadIdx.x & 3)) & 1u) ? 0.f : -INFINITY;
  // zero the rows of Q that TMA never writes: rows 12R..127 (prefill), or rows 32q+12..32q+31
  // of every lane quarter q (decode: the 12 head rows are loaded at rows 32q..32q+11)
  {
    const int box_rows = kGroup * R;
    const int pad_rows = kDec ? 4 * (32 - kGroup) : 128 - box_rows;
    for (int i = threadIdx.x; i < pad_rows * 16; i += blockDim.x) {
      const int pr = i / 16, c = i % 16;   // 16 x 16 B per row (both panels)
      const int r = kDec ? (pr / (32 - kGroup)) * 32 + kGroup + pr % (32 - kGroup) : box_rows + pr;
      const int panel = c / 8, cc = c % 8;
      *reinterpret_cast<uint4*>(sQ + panel * 16384 + r * 128 + cc * 16) = make_uint4(0, 0, 0, 0);
    }
    fence_proxy_async_smem();
  }
  if (warp == C::kMmaWarp) {
    tmem_alloc(s_tmem, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;
  const uint32_t tmem_O = tmem + 256;

  const int32_t* uni = rec + args.pl.union_off();
  const uint32_t* masks = reinterpret_cast<const uint32_t*>(rec + args.pl.mask_off());
  const int mwords = args.pl.umax / 32;
  const int col0 = kDec ? 0 : g * kHeadDim;
  // P: its own columns [384, 512), two buffers of 64 (bf16 pairs)
  const uint32_t tmem_P = tmem + 384;
  constexpr int kPStride = 64;

  if (warp >= C::kSoftWarps) {
  // the last two warpgroups (MMA and producers) give registers up for the softmax warpgroups
  regs_lower<C::kRegsOther>();
  if (warp >= C::kKWarp0 && warp < C::kKWarp0 + C::kKWarps) {
    // ---------------- Q + K producers ----------------
    const int kw = warp - C::kKWarp0;
    if (kw == 0 && lane == 0) {
      prefetch_tmap(&maps.q);
      for (int j = 0; j < kNumBoxSizes; ++j) prefetch_tmap(&maps.k[j]);
      const uint32_t qbytes = 2u * kGroup * R * 128u;   // full box, out-of-range rows zero-filled
      constexpr int kCopies = kDec ? 4 : 1;            // decode: one copy per lane quarter
      mbar_arrive_expect_tx(q_full, kCopies * qbytes);
      for (int cp = 0; cp < kCopies; ++cp)
        for (int half = 0; half < 2; ++half)
          tma_load_3d(sQ + half * 16384 + cp * 4096, &maps.q, half * 64, g * kGroup,
                      static_cast<int32_t>(tok_row0), q_full);
    }
    __syncwarp();
    attn_producer<kPaged>(maps.k, sK, k_full, k_empty, C::kKStages, uni, U, c_begin, nchunks,
                  kv_row_base, col0, args.oob_row, args.pg, tile, g, kw, C::kKWarps, s_abort,
                  args.st, 20, fault);
    if (kw == 0 && lane == 0 && *s_abort) mbar_drain(q_full, 0);
  } else if (warp >= C::kVWarp0) {
    // ---------------- V producers ----------------
    const int vw = warp - C::kVWarp0;
    if (vw == 0 && lane == 0)
      for (int j = 0; j < kNumBoxSizes; ++j) prefetch_tmap(&maps.v[j]);
    __syncwarp();
    attn_producer<kPaged>(maps.v, sV, v_full, v_empty, C::kVStages, uni, U, c_begin, nchunks,
                  kv_row_base, col0, args.oob_row, args.pg, tile, g, vw, C::kVWarps, s_abort,
                  args.st, 27, false);
  } else {
    // ---------------- MMA issuer (warp kMmaWarp) ----------------
    if (lane == 0) {
      const uint32_t sQ0 = smem_u32(sQ);
      const uint64_t lim = fault ? kFaultWaitNs : kWaitLimitNs;
      bool ok = mbar_wait(q_full, 0, s_abort, args.st, 21, lim);
      auto issue_pv = [&](int j) -> bool {
        const int bj = j & 1;
        const int vs = j % C::kVStages;
        if (!mbar_wait(&p_full[bj], (j >> 1) & 1, s_abort, args.st, 22, lim)) return false;
        if (!mbar_wait(&v_full[vs], (j / C::kVStages) & 1, s_abort, args.st, 28, lim)) return false;
        tc_fence_after();
        const uint32_t sV0 = smem_u32(sV + vs * C::kKVBytes);
#pragma unroll
        for (int k = 0; k < C::kChunkKeys / 16; ++k) {
          // B = V chunk, MN-major: 16 keys per step = 2048 bytes; next 64 dims at +16 KB
          const uint64_t db = smem_desc_sw128(sV0 + 2048 * k, 16384, 1024);
          umma_ts(tmem_O, tmem_P + bj * kPStride + 8 * k, db, C::kIdescPV,
                  (j > 0 || k > 0) ? 1u : 0u);
        }
        umma_commit(&v_empty[vs]);
        umma_commit(&p_free[bj]);
        umma_commit(pv_done);
        return true;
      };
      for (int i = 0; ok && i < nchunks; ++i) {
        const int b = i & 1;
        const int ks = i % C::kKStages;
        if (!mbar_wait(&k_full[ks], (i / C::kKStages) & 1, s_abort, args.st, 23, lim)) break;
        // S_i overwrites S_{i-2}, which the softmax finished reading before it arrived on
        // p_full for chunk i-2 (waited for when P_{i-2}.V was issued).  P has its own columns,
        // which no S MMA touches; the softmax rewrites P of this buffer only after s_full of
        // chunk i, whose commit also covers P_{i-2}.V.  Decode keeps the stricter order (S_i
        // after P_{i-2}.V has completed).
        if (kDec && i >= 2 && !mbar_wait(&p_free[b], ((i - 2) >> 1) & 1, s_abort, args.st, 29, lim))
          break;
        tc_fence_after();
        const uint32_t sK0 = smem_u32(sK + ks * C::kKVBytes);
#pragma unroll
        for (int k = 0; k < kHeadDim / 16; ++k) {
          const int half = k >> 2, kk = k & 3;
          const uint64_t da = smem_desc_sw128(sQ0 + half * 16384 + 32 * kk, 0, 1024);
          const uint64_t db = smem_desc_sw128(sK0 + half * 16384 + 32 * kk, 0, 1024);
          umma_ss(tmem + b * 128, da, db, C::kIdescQK, k > 0 ? 1u : 0u);
        }
        umma_commit(&k_empty[ks]);
        umma_commit(&s_full[b]);
        if (i > 0 && !issue_pv(i - 1)) break;
        if (i == nchunks - 1 && issue_pv(i)) umma_commit(o_final);
      }
      umma_commit(mma_done);
      mbar_drain(mma_done, 0);
    }
  }
  } else {
    regs_raise<C::kRegsSoftmax>();
    if constexpr (kDec) {
      // ---------------- decode softmax (warps 0 .. 7) ----------------
      // One query token: its 12 head rows sit in every lane quarter (rows 32q .. 32q+11 hold
      // copy q), so all eight softmax warps hold valid rows.  Copy q owns keys 16q..16q+15 of
      // each warpgroup's 64-key half of every chunk and keeps its own running max and sum:
      // P of a row is zero outside its copy's keys (P lives in its own TMEM columns, zeroed
      // once; a thread rewrites only its 16 keys), so O row 32q+h accumulates copy q's part
      // of head h.  The four partial softmaxes are merged by log-sum-exp at the end.  Row
      // maxima are shared between the two warpgroups as in prefill.
      static_assert(C::kSoftGroups == 2, "decode softmax assumes two warpgroups");
      const int wg = warp >> 2;
      const int quarter = warp & 3;
      const int row = quarter * 32 + lane;
      const bool row_ok = lane < kGroup;
      const int cs = 64 * wg + 16 * quarter;   // my first key column of a chunk
      const int bs = cs / kBlock;              // my first block slot of a chunk
      const int tail_u = rec[args.pl.tail_off()];
      const int tail_last = pos0 % kBlock;
      const float sl2 = 1.4426950408889634f * 0.08838834764831845f;   // log2(e)/sqrt(128)
      float m = -INFINITY, l = 0.f;
      const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
      {
        uint32_t z[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) z[j] = 0u;
        tmem_st32(tmem_P + lane_base + 32 * wg, z);
        tmem_st32(tmem_P + lane_base + kPStride + 32 * wg, z);
        tmem_wait_st();
      }
      uint32_t mword_next = masks[c_begin];
      bool ok = true;
      for (int i = 0; i < nchunks; ++i) {
        const int b = i & 1;
        const int q = c_begin + i;
        const uint32_t mword = row_ok ? (mword_next >> bs) & 0xFu : 0u;
        if (i + 1 < nchunks) mword_next = masks[q + 1];
        bool got = ok ? mbar_wait(&s_full[b], (i >> 1) & 1, s_abort, args.st, 24) : false;
        if (__any_sync(0xffffffffu, !got)) ok = false;
        tc_fence_after();
        uint32_t sv[16];
        float mx = -INFINITY;
        if (ok) {
          tmem_ld16(tmem + lane_base + b * 128 + cs, sv);
          tmem_wait_ld();
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const float bias = ((mword >> u) & 1u) ? 0.f : -INFINITY;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              sv[4 * u + kk] = __float_as_uint(__uint_as_float(sv[4 * u + kk]) + bias);
          }
          // the own block: hide the tokens after the query (only where it lies)
          const int tu = tail_u - q * C::kChunkBlocks - bs;
          if (tu >= 0 && tu < 4) {
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              if (u == tu) {
                if (tail_last < 1) sv[4 * u + 1] = __float_as_uint(-INFINITY);
                if (tail_last < 2) sv[4 * u + 2] = __float_as_uint(-INFINITY);
                if (tail_last < 3) sv[4 * u + 3] = __float_as_uint(-INFINITY);
              }
            }
          }
          float mxs[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) mxs[j] = __uint_as_float(sv[j]);
#pragma unroll
          for (int j = 4; j < 16; ++j) mxs[j & 3] = fmaxf(mxs[j & 3], __uint_as_float(sv[j]));
          mx = fmaxf(fmaxf(mxs[0], mxs[1]), fmaxf(mxs[2], mxs[3]));
        }
        xmax[(b * 2 + wg) * 128 + row] = mx;
        tc_fence_before();
        named_barrier_sync(2 + quarter, 64);   // the two warps holding this lane quarter's rows
        tc_fence_after();
        if (ok) {
          mx = fmaxf(mx, xmax[(b * 2 + (wg ^ 1)) * 128 + row]);
          const float m_cand = fmaxf(m, mx * sl2);
          const bool need = m_cand > m + 8.f || (m == -INFINITY && m_cand > -INFINITY);
          const bool rescale = __any_sync(0xffffffffu, need);
          float alpha = 1.f;
          if (rescale) {
            alpha = (m == -INFINITY) ? 0.f : ex2_approx(m - m_cand);
            m = m_cand;
          }
          const float mneg = (m == -INFINITY) ? 0.f : -m;
          uint32_t pv[8];
          float lsum[2] = {0.f, 0.f};
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const float p0 = ex2_approx(fmaf(__uint_as_float(sv[2 * j]), sl2, mneg));
            const float p1 = ex2_approx(fmaf(__uint_as_float(sv[2 * j + 1]), sl2, mneg));
            lsum[j & 1] += p0 + p1;
            pv[j] = pack_bf16x2(p0, p1);
          }
          l = l * alpha + (lsum[0] + lsum[1]);
          tmem_st8(tmem_P + lane_base + b * kPStride + cs / 2, pv);
          tmem_wait_st();
          if (rescale && i > 0) {
            // as in prefill: wait until P.V of chunk i-1 is in O, then rescale my dims
            const bool gotpv = mbar_wait(pv_done, (i - 1) & 1, s_abort, args.st, 25);
            if (__any_sync(0xffffffffu, !gotpv)) ok = false;
            if (ok) {
              tc_fence_after();
              const uint32_t to = tmem_O + lane_base + 64 * wg;
#pragma unroll
              for (int c = 0; c < 2; ++c) {
                uint32_t ov[32];
                tmem_ld32(to + 32 * c, ov);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 32; ++j) ov[j] = __float_as_uint(__uint_as_float(ov[j]) * alpha);
                tmem_st32(to + 32 * c, ov);
              }
              tmem_wait_st();
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[b]);
      }
      // merge: each copy's (max, sum, unnormalised O row) goes to shared memory (the K ring is
      // idle once every P.V has completed), then 192 threads each combine 8 dims of one head
      xsum[wg * 128 + row] = l;
      named_barrier_sync(1, 256);
      const float l_all = xsum[row] + xsum[128 + row];
      float* mo = reinterpret_cast<float*>(sK);          // [copy][head][128]
      float* mm = xmax;                                  // [copy][head]: max (log2 domain)
      float* ml = xmax + 4 * kGroup;                     // [copy][head]: sum
      const bool got = ok ? mbar_wait(o_final, 0, s_abort, args.st, 26) : false;
      if (!__any_sync(0xffffffffu, !got)) {
        tc_fence_after();
        uint32_t ov[64];
        tmem_ld32(tmem_O + lane_base + 64 * wg, ov);
        tmem_ld32(tmem_O + lane_base + 64 * wg + 32, ov + 32);
        tmem_wait_ld();
        if (row_ok) {
          const int cr = quarter * kGroup + lane;
          float4* dst = reinterpret_cast<float4*>(mo + cr * kHeadDim + 64 * wg);
#pragma unroll
          for (int c = 0; c < 16; ++c)
            dst[c] = make_float4(__uint_as_float(ov[4 * c]), __uint_as_float(ov[4 * c + 1]),
                                 __uint_as_float(ov[4 * c + 2]), __uint_as_float(ov[4 * c + 3]));
          if (wg == 0) {
            mm[cr] = m;
            ml[cr] = l_all;
          }
        }
      } else {
        ok = false;
      }
      named_barrier_sync(1, 256);
      const int t = threadIdx.x;
      if (t < kGroup * 16) {
        const int h = t / 16, d0 = (t % 16) * 8;
        float M = -INFINITY;
#pragma unroll
        for (int c = 0; c < 4; ++c) M = fmaxf(M, mm[c * kGroup + h]);
        float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        float L = 0.f;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const float mc = mm[c * kGroup + h];
          const float f = (mc == -INFINITY) ? 0.f : ex2_approx(mc - M);
          L += f * ml[c * kGroup + h];
          const float4* src = reinterpret_cast<const float4*>(mo + (c * kGroup + h) * kHeadDim + d0);
          const float4 a0 = src[0], a1 = src[1];
          acc[0] += f * a0.x; acc[1] += f * a0.y; acc[2] += f * a0.z; acc[3] += f * a0.w;
          acc[4] += f * a1.x; acc[5] += f * a1.y; acc[6] += f * a1.z; acc[7] += f * a1.w;
        }
        if (args.splits == 1 && !args.partials) {
          const float inv = L > 0.f ? 1.f / L : 0.f;
          uint4 v;
          v.x = pack_bf16x2(acc[0] * inv, acc[1] * inv);
          v.y = pack_bf16x2(acc[2] * inv, acc[3] * inv);
          v.z = pack_bf16x2(acc[4] * inv, acc[5] * inv);
          v.w = pack_bf16x2(acc[6] * inv, acc[7] * inv);
          *reinterpret_cast<uint4*>(args.out + (tok_row0 * kHeads + g * kGroup + h) * kHeadDim +
                                    d0) = v;
        } else {
          const int64_t pr =
              ((static_cast<int64_t>(tile) * 2 + g) * args.splits + split) * kGroup + h;
          if (d0 == 0) {
            args.part_m[pr] = M;
            args.part_l[pr] = L;
          }
          float4* po = reinterpret_cast<float4*>(args.part_o + pr * kHeadDim + d0);
          po[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
          po[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
        }
      }
    } else {
      // ---------------- softmax (warps 0 .. 4 kSoftGroups - 1) ----------------
      // kSoftGroups warpgroups share each row: group sg handles keys [kCols sg, kCols (sg + 1))
      // of every chunk and dims [kCols sg, ...) of O.  Row maxima are exchanged through shared
      // memory (double-buffered by chunk parity, one named barrier per chunk and lane quarter,
      // ids 2..5); partial row sums are combined once at the end.  All groups take identical
      // rescale decisions.
      // A warp's 32 rows belong to about three tokens: the exponentials of each pair of blocks
      // that none of them attends are skipped (a warp-uniform branch) and its P is left zero,
      // about half of the union's blocks on long rows.  The block mask is applied once per
      // block: to the block's maximum, and as an exponent offset of -inf for the blocks the
      // row's token did not select (a bias added to every key cost 6% more time).  The softmax
      // is bound mostly by its instruction stream: most instructions taken out of a chunk
      // showed in the kernel's time.
      static_assert(C::kSoftGroups == 2, "prefill softmax assumes two warpgroups");
      constexpr int kSG = C::kSoftGroups;
      constexpr int kCols = 128 / kSG;              // keys (and O dims) per group
      constexpr int kBlk = kCols / kBlock;          // blocks per group
      const int wg = warp >> 2;
      const int quarter = warp & 3;           // TMEM lanes 32q .. 32q+31
      const int row = quarter * 32 + lane;
      const int valid_rows = kGroup * ntok;
      const bool row_ok = row < valid_rows;
      const bool warp_active = quarter * 32 < valid_rows;
      const int tr = row_ok ? row / kGroup : 0;
      const int hr = row % kGroup;
      const int pos = pos0 + tr;
      const int tail_u = row_ok ? rec[args.pl.tail_off() + tr] : -1000000;
      const int tail_last = pos % kBlock;   // keys 0..tail_last of the own block are visible
      const float sl2 = 1.4426950408889634f * 0.08838834764831845f;   // log2(e)/sqrt(128)
      float m = -INFINITY, l = 0.f;
      const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
      const uint32_t* mrow = masks + tr * mwords;
      uint32_t mword_next = row_ok ? mrow[c_begin] : 0u;
      const float4* lut4 = reinterpret_cast<const float4*>(smem + C::kLutOff);
      bool ok = true;
      for (int i = 0; i < nchunks; ++i) {
        const int b = i & 1;
        const int q = c_begin + i;
        const uint32_t mword = (mword_next >> (kBlk * wg)) & ((1u << kBlk) - 1u);   // my blocks
        const uint32_t warp_need = __reduce_or_sync(0xffffffffu, mword);   // blocks any row of the warp attends
        if (row_ok && i + 1 < nchunks) mword_next = mrow[q + 1];
        bool got = ok ? mbar_wait(&s_full[b], (i >> 1) & 1, s_abort, args.st, 24) : false;
        if (__any_sync(0xffffffffu, !got)) ok = false;   // also reconverges the warp
        tc_fence_after();
        uint32_t sv[kCols];
        const uint32_t ts = tmem + lane_base + b * 128;
        float mx = -INFINITY;
        // 0 / -inf per block of this row's token, four blocks per table read (a bit test and a
        // select per block cost 1.7% more time)
        float bias[kBlk];
  #pragma unroll
        for (int n = 0; n < kBlk / 4; ++n) {
          const float4 bb = lut4[(mword >> (4 * n)) & 15u];
          bias[4 * n] = bb.x; bias[4 * n + 1] = bb.y; bias[4 * n + 2] = bb.z; bias[4 * n + 3] = bb.w;
        }
        if (ok && warp_active) {
  #pragma unroll
          for (int c = 0; c < kCols / 32; ++c) tmem_ld32(ts + kCols * wg + 32 * c, sv + 32 * c);
          tmem_wait_ld();
          // the own block: hide the tokens after the query (only where it lies).  Selects, not
          // branches on u == tu: the branches made the compiler spill S to local memory.
          const int tu = tail_u - q * C::kChunkBlocks - kBlk * wg;
          if (__any_sync(0xffffffffu, tu >= 0 && tu < kBlk)) {
  #pragma unroll
            for (int u = 0; u < kBlk; ++u) {
              const bool own = u == tu;
              sv[4 * u + 1] = (own && tail_last < 1) ? __float_as_uint(-INFINITY) : sv[4 * u + 1];
              sv[4 * u + 2] = (own && tail_last < 2) ? __float_as_uint(-INFINITY) : sv[4 * u + 2];
              sv[4 * u + 3] = (own && tail_last < 3) ? __float_as_uint(-INFINITY) : sv[4 * u + 3];
            }
          }
          // each block's maximum, -inf for the blocks this row's token did not select
          float bm[kBlk];
  #pragma unroll
          for (int u = 0; u < kBlk; ++u) {
            bm[u] = fmaxf(fmaxf(__uint_as_float(sv[4 * u]), __uint_as_float(sv[4 * u + 1])),
                          fmaxf(__uint_as_float(sv[4 * u + 2]), __uint_as_float(sv[4 * u + 3]))) + bias[u];
          }
          static_assert(kBlk == 16, "a four-level tree");
  #pragma unroll
          for (int u = 0; u < 8; ++u) bm[u] = fmaxf(bm[u], bm[u + 8]);
  #pragma unroll
          for (int u = 0; u < 4; ++u) bm[u] = fmaxf(bm[u], bm[u + 4]);
          mx = fmaxf(fmaxf(bm[0], bm[2]), fmaxf(bm[1], bm[3]));
        }
        // exchange the partial row maxima (every softmax warp takes part, active or not)
        xmax[(b * kSG + wg) * 128 + row] = mx;
        tc_fence_before();
        // only the two warps of this lane quarter (they share its rows) meet here: a barrier
        // over all eight softmax warps cost 0.8% more time
        named_barrier_sync(2 + quarter, 32 * kSG);
        tc_fence_after();
        if (ok && warp_active) {
  #pragma unroll
          for (int o = 1; o < kSG; ++o) mx = fmaxf(mx, xmax[(b * kSG + ((wg + o) % kSG)) * 128 + row]);
          const float m_cand = fmaxf(m, mx * sl2);
          // lazy rescale: P may reach 2^16 (bf16 keeps its relative precision; O and the sum are
          // fp32), so O is rescaled only when a row's maximum grows by more than 16 (log2 units)
          const bool grow = m_cand > m + 16.f || (m == -INFINITY && m_cand > -INFINITY);
          const bool rescale = __any_sync(0xffffffffu, grow);
          float alpha = 1.f;
          if (rescale) {
            alpha = (m == -INFINITY) ? 0.f : ex2_approx(m - m_cand);
            m = m_cand;
          }
          const float mneg = (m == -INFINITY) ? 0.f : -m;
          // P overwrites S in registers: packed pair j lands in sv[j], whose S value (key j) was
          // consumed at pair j/2 <= j
          uint64_t lsum2[2] = {0ull, 0ull};   // row sums as packed pairs (add.rn.f32x2)
          constexpr int kSk = 2;                 // blocks per skip decision (1, 2, 4: 2 measured best)
  #pragma unroll
          for (int gi = 0; gi < kBlk / kSk; ++gi) {
            if ((warp_need >> (gi * kSk)) & ((1u << kSk) - 1u)) {
  #pragma unroll
              for (int jj = 0; jj < 2 * kSk; ++jj) {
                const int j = gi * 2 * kSk + jj;
                // blocks the row's token did not select: exponent -inf, so P = 0
                const float off = mneg + bias[j >> 1];
                // the pair's exponent arguments on one packed fma.rn.f32x2 (1.2% less time)
                const uint64_t x = f2_fma(f2_pack(__uint_as_float(sv[2 * j]), __uint_as_float(sv[2 * j + 1])),
                                          f2_pack(sl2, sl2), f2_pack(off, off));
                const float p0 = ex2_approx(f2_lo(x));
                const float p1 = ex2_approx(f2_hi(x));
                lsum2[j & 1] = f2_add(lsum2[j & 1], f2_pack(p0, p1));
                sv[j] = pack_bf16x2(p0, p1);
              }
            } else {
  #pragma unroll
              for (int jj = 0; jj < 2 * kSk; ++jj) sv[gi * 2 * kSk + jj] = 0u;
            }
          }
          const uint64_t ls = f2_add(lsum2[0], lsum2[1]);
          l = l * alpha + (f2_lo(ls) + f2_hi(ls));
          // packed P of my keys -> columns kCols/2 sg .. of this buffer's P (P.V of chunk i-2,
          // which last read them, completed before S_i: one commit tracks every earlier MMA)
          tmem_st32(tmem_P + lane_base + b * kPStride + 32 * wg, sv);
          tmem_wait_st();
          if (rescale && i > 0) {
            // O holds P.V of chunks < i-1 and maybe i-1: wait until chunk i-1 is in, rescale
            // my dims of O.  P.V of chunk i cannot start before this warp arrives on p_full.
            const bool gotpv = mbar_wait(pv_done, (i - 1) & 1, s_abort, args.st, 25);
            if (__any_sync(0xffffffffu, !gotpv)) ok = false;
            if (ok) {
              tc_fence_after();
              const uint32_t to = tmem_O + lane_base + kCols * wg;
  #pragma unroll
              for (int c = 0; c < kCols / 32; ++c) {
                uint32_t ov[32];
                tmem_ld32(to + 32 * c, ov);
                tmem_wait_ld();
  #pragma unroll
                for (int j = 0; j < 32; ++j) ov[j] = __float_as_uint(__uint_as_float(ov[j]) * alpha);
                tmem_st32(to + 32 * c, ov);
              }
              tmem_wait_st();
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[b]);
      }
      // combine the partial row sums
      xsum[wg * 128 + row] = l;
      named_barrier_sync(1, 128 * kSG);
      float l_all = 0.f;
  #pragma unroll
      for (int o = 0; o < kSG; ++o) l_all += xsum[o * 128 + row];
      if (ok && nchunks > 0) {
        // a dedicated barrier: two P.V may still be in flight here, so a parity wait on
        // pv_done could match an older phase
        const bool got = mbar_wait(o_final, 0, s_abort, args.st, 26);
        if (!__any_sync(0xffffffffu, !got)) {
          tc_fence_after();
          if (warp_active) {
            const uint32_t to = tmem_O + lane_base + kCols * wg;
            uint32_t ov[kCols];
  #pragma unroll
            for (int c = 0; c < kCols / 32; ++c) tmem_ld32(to + 32 * c, ov + 32 * c);
            tmem_wait_ld();
            if (row_ok) {
              if (!kDec || args.splits == 1) {   // one split: the final output directly
                const float inv = l_all > 0.f ? 1.f / l_all : 0.f;
                __nv_bfloat16* o = args.out + ((tok_row0 + tr) * kHeads + g * kGroup + hr) * kHeadDim +
                                   kCols * wg;
  #pragma unroll
                for (int c = 0; c < kCols / 8; ++c) {
                  uint4 v;
                  v.x = pack_bf16x2(__uint_as_float(ov[8 * c + 0]) * inv, __uint_as_float(ov[8 * c + 1]) * inv);
                  v.y = pack_bf16x2(__uint_as_float(ov[8 * c + 2]) * inv, __uint_as_float(ov[8 * c + 3]) * inv);
                  v.z = pack_bf16x2(__uint_as_float(ov[8 * c + 4]) * inv, __uint_as_float(ov[8 * c + 5]) * inv);
                  v.w = pack_bf16x2(__uint_as_float(ov[8 * c + 6]) * inv, __uint_as_float(ov[8 * c + 7]) * inv);
                  reinterpret_cast<uint4*>(o)[c] = v;
                }
              } else {
                const int64_t pr =
                    ((static_cast<int64_t>(tile) * 2 + g) * args.splits + split) * kGroup + hr;
                if (wg == 0) {
                  args.part_m[pr] = m;
                  args.part_l[pr] = l_all;
                }
                float4* po = reinterpret_cast<float4*>(args.part_o + pr * kHeadDim + kCols * wg);
  #pragma unroll
                for (int c = 0; c < kCols / 4; ++c)
                  po[c] = make_float4(__uint_as_float(ov[4 * c]), __uint_as_float(ov[4 * c + 1]),
                                      __uint_as_float(ov[4 * c + 2]), __uint_as_float(ov[4 * c + 3]));
              }
            }
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == C::kMmaWarp) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

}  // namespace qsa
