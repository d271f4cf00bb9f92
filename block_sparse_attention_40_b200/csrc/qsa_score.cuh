// qsa_score.cuh -- step a2, the MQA indexer score, on tcgen05 tensor cores.
//
//   s(t, b) = sum_h w[t,h] * ReLU(q_idx[t,h] . kbar[b])      (16 heads, width 64)
//
// A dense contraction: D[block, (token, head)] = kbar[block, :] . q_idx[(token, head), :]
// with M = 128 compressed blocks per tile (A operand, streamed by TMA), N = 16 tokens x 16
// heads = 256 (prefill) or 1 token x 16 heads (decode) (B operand, loaded once per CTA),
// K = 64.  The fp32 accumulator lives in TMEM (two buffers, so the epilogue of tile i
// overlaps the MMA of tile i+1).  Epilogue: each thread owns one block row, reads its
// 16 heads per token from TMEM (prefill: four tokens, read as two pairs so that the second
// read overlaps the sums of the first), applies ReLU, weights by w and sums in fp32 (even and
// odd heads as two partial sums), and writes the score if the block is a candidate of that
// token (b < floor(pos/4)).
//
// Warp roles: warp 0 issues TMA, warp 1 allocates TMEM and issues MMAs (one thread),
// the remaining warps run the epilogue.

#pragma once

#include "qsa_common.cuh"
#include "qsa_misc.cuh"

namespace qsa {

template <int NTOK>
struct ScoreCfg {
  static constexpr int kN = NTOK * kIdxHeads;             // MMA N
  static constexpr int kAccCols = kN < 32 ? 32 : kN;      // TMEM columns per accumulator
  static constexpr int kNumAcc = NTOK == 16 ? 2 : 4;
  static constexpr int kTmemCols = kAccCols * kNumAcc;    // 512 / 128
  static constexpr int kStages = NTOK == 16 ? 4 : 5;     // decode: 2 CTAs per SM
  static constexpr int kCtasPerSm = NTOK == 16 ? 1 : 2;
  static constexpr int kEpiWarps = NTOK == 16 ? 16 : 4;   // prefill: 4 token groups x 4 lane quarters
  static constexpr int kThreads = 64 + 32 * kEpiWarps;
  static constexpr int kABytes = 128 * kIdxDim * 2;       // 16 KB
  static constexpr int kBBytes = kN * kIdxDim * 2;        // 32 KB / 2 KB
  static constexpr int kBOff = kStages * kABytes;
  static constexpr int kWOff = kBOff + ((kBBytes + 1023) / 1024) * 1024;
  static constexpr int kBarOff = kWOff + NTOK * kIdxHeads * 4;
  static constexpr int kNumBars = 2 * kStages + 2 * kNumAcc + 2;
  // decode: first-digit (key bits 31..20) histogram of this CTA's scores, flushed to global
  static constexpr int kHistOff = kBarOff + kNumBars * 8 + 16;
  static constexpr int kHistBytes = NTOK == 1 ? 4096 * 4 : 0;
  static constexpr int kSmemBytes = kHistOff + kHistBytes + 1024;  // + align slack
  // prefill with select_mode 1: each token row's first-digit histogram, 4096 16-bit counters
  // packed in pairs, at kHistOff
  static constexpr int kRowHistWords = 2048;
  static constexpr int kSmemBytesFused = kHistOff + NTOK * kRowHistWords * 4 + 1024;
  static constexpr uint32_t kIdesc = idesc_bf16_f32(128, kN, 0, 0);
  static_assert(kCtasPerSm * (kSmemBytes + 1024) <= 228 * 1024, "shared memory per SM");
  static_assert(kCtasPerSm * kTmemCols <= 512, "TMEM columns per SM");
  static_assert(NTOK != 16 || kSmemBytesFused <= 227 * 1024, "shared memory per CTA");
};

struct ScoreArgs {
  // prefill
  const SeqMeta* meta;
  int32_t num_seqs;
  int32_t tile_begin;      // global 16-token tile range [tile_begin, tile_begin + gridDim.x)
  int32_t tile_count;
  int32_t topk_skip;       // skip tiles whose largest n_c <= topk_skip (0 = none)
  int64_t row_begin;       // score row 0 corresponds to this global token
  // decode
  const int32_t* len;      // [B]
  int32_t splits;
  int32_t mtiles_per_split;
  int64_t kbar_rows_per_seq;
  Paging pg;               // where each sequence's compressed keys live (table null: contiguous)
  int32_t kbar_oob_row;    // a row past the compressed-key pool (TMA reads it as zeros)
  int32_t* n_c_out;        // [B] n_c per sequence (written by split 0), may be null
  // decode of one shard of a longer context: the cache holds the sequence's tokens from
  // global block block0 on, glen [B] holds the sequences' whole lengths (null: not a shard)
  const int32_t* glen;
  int32_t block0;
  uint32_t* hist;          // [B][4096] first-digit histograms of the scores (zeroed), or null
  // prefill with select_mode 1: per score row, the first-digit threshold bin of its top-k, as
  // rinfo[4 r] = bin, [4 r + 1] = keys in higher bins, [4 r + 2] = keys in the bin (rows with
  // more candidates than the budget; null: not built)
  int32_t* rinfo;
  int32_t topk;
  // common
  const __nv_bfloat16* w;  // prefill: [T][16]; decode: [B][16]
  float* scores;
  int64_t ld;
  DevStatus st;
};

template <int NTOK>
struct ScoreWork {
  int64_t a_row0;    // first kbar row of this CTA's first M-tile
  int32_t mt0;       // first M-tile index (block offset = 128 * (mt0 + i))
  int32_t n_mtiles;
  int32_t b_row0;    // first q_idx row (token * 16)
  int32_t ntok;      // valid tokens in the N tile
  int32_t pos0;      // position (within the sequence) of token 0
  int64_t out_row0;  // score row of token 0
  int32_t seq;       // decode: the sequence
  int32_t n_c;       // decode: candidate blocks (local to the cache) of the sequence
};

// s = sum_h w[h] * ReLU(d[h]) over the 16 heads of one (token, block): the even and the odd
// heads accumulate as the two halves of packed f32x2 FMAs (each an fp32 fused multiply-add),
// and the two partial sums are added at the end.  w: 16 weights in shared memory, 16-byte
// aligned; d: the 16 fp32 accumulator words read from TMEM.
__device__ __forceinline__ float head_weighted_relu_sum(const uint32_t* d, const float* w) {
  const float4* w4 = reinterpret_cast<const float4*>(w);
  uint64_t acc = 0ull;   // (+0.f, +0.f)
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const float4 wq = w4[q];
    uint64_t wa, wb, ra, rb;
    asm("mov.b64 %0, {%1, %2};" : "=l"(wa) : "f"(wq.x), "f"(wq.y));
    asm("mov.b64 %0, {%1, %2};" : "=l"(wb) : "f"(wq.z), "f"(wq.w));
    asm("mov.b64 %0, {%1, %2};" : "=l"(ra)
        : "f"(fmaxf(__uint_as_float(d[4 * q]), 0.f)), "f"(fmaxf(__uint_as_float(d[4 * q + 1]), 0.f)));
    asm("mov.b64 %0, {%1, %2};" : "=l"(rb)
        : "f"(fmaxf(__uint_as_float(d[4 * q + 2]), 0.f)), "f"(fmaxf(__uint_as_float(d[4 * q + 3]), 0.f)));
    asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(acc) : "l"(wa), "l"(ra));
    asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(acc) : "l"(wb), "l"(rb));
  }
  float even, odd;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(even), "=f"(odd) : "l"(acc));
  return even + odd;
}

template <int NTOK>
__device__ __forceinline__ ScoreWork<NTOK> score_work(const ScoreArgs& a) {
  ScoreWork<NTOK> wk;
  if constexpr (NTOK == 16) {
    const int gt = a.tile_begin + (a.tile_count - 1 - static_cast<int>(blockIdx.x));
    const int s = find_seq_of_tile<false>(a.meta, a.num_seqs, gt);
    const SeqMeta m = a.meta[s];
    const int lt = gt - m.score_tile0;
    const int p0 = lt * 16;
    const int ntok = (m.len - p0) < 16 ? (m.len - p0) : 16;
    const int c_max = (p0 + ntok - 1) / kBlock;
    wk.ntok = ntok;
    wk.pos0 = p0;
    wk.mt0 = 0;
    wk.n_mtiles = (ntok <= 0 || c_max <= a.topk_skip) ? 0 : (c_max + 127) / 128;
    wk.a_row0 = m.kbar0;
    wk.b_row0 = static_cast<int32_t>((m.tok0 + p0) * kIdxHeads);
    wk.out_row0 = m.tok0 + p0 - a.row_begin;
    wk.seq = s;
    wk.n_c = 0;   // per token: floor(pos / 4)
  } else {
    const int b = static_cast<int>(blockIdx.x) / a.splits;
    const int split = static_cast<int>(blockIdx.x) % a.splits;
    int p, n_c;
    if (a.glen != nullptr) {
      // a shard: the candidates are the shard's complete blocks before the query's own block
      p = a.glen[b] - 1;
      const int own = p >= 0 ? p / kBlock : 0;
      n_c = own - a.block0;
      const int here = a.len[b] / kBlock;
      n_c = n_c < 0 ? 0 : (n_c > here ? here : n_c);
    } else {
      p = a.len[b] - 1;
      n_c = p >= 0 ? p / kBlock : 0;
    }
    // The grid covers the blocks of the host lengths the caller passed.  A device length
    // beyond them (a stale host copy) is reported, and only the covered blocks are scored;
    // the top-k then sees that same count, so it never reads a score that was not written.
    const int covered = a.splits * a.mtiles_per_split * 128;
    if (n_c > covered) {
      if (split == 0 && threadIdx.x == 0) report_error(a.st, kErrDevice, 207);
      n_c = covered;
    }
    if (split == 0 && threadIdx.x == 0 && a.n_c_out) a.n_c_out[b] = n_c;
    const int total = (n_c + 127) / 128;
    const int m0 = split * a.mtiles_per_split;
    int m1 = m0 + a.mtiles_per_split;
    if (m1 > total) m1 = total;
    wk.ntok = 1;
    wk.pos0 = p;
    wk.mt0 = m0;
    wk.n_mtiles = m1 > m0 ? m1 - m0 : 0;
    wk.a_row0 = static_cast<int64_t>(b) * a.kbar_rows_per_seq;
    wk.b_row0 = b * kIdxHeads;
    wk.out_row0 = b;
    wk.seq = b;
    wk.n_c = n_c;
  }
  return wk;
}

// kRowHist (prefill, select_mode 1): also count each token row's first-digit histogram and
// find its threshold bin (args.rinfo); a separate instantiation, so the default path carries
// none of it.
template <int NTOK, bool kRowHist = false>
__global__ void __launch_bounds__(ScoreCfg<NTOK>::kThreads, ScoreCfg<NTOK>::kCtasPerSm)
    k_index_score(const __grid_constant__ CUtensorMap tmap_kbar,
                  const __grid_constant__ CUtensorMap tmap_qidx, ScoreArgs args) {
  using C = ScoreCfg<NTOK>;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  unsigned char* sA = smem;
  unsigned char* sB = smem + C::kBOff;
  float* sW = reinterpret_cast<float*>(smem + C::kWOff);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
  uint64_t* full = bars;
  uint64_t* empty = bars + C::kStages;
  uint64_t* acc_full = bars + 2 * C::kStages;
  uint64_t* acc_empty = acc_full + C::kNumAcc;
  uint64_t* b_full = acc_empty + C::kNumAcc;
  uint64_t* mma_done = b_full + 1;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(bars + C::kNumBars);
  volatile int* s_abort = reinterpret_cast<volatile int*>(s_tmem + 1);

  pdl_trigger();
  pdl_wait();   // decode: the lengths, keys and weights come from earlier kernels
  const ScoreWork<NTOK> wk = score_work<NTOK>(args);
  if (wk.n_mtiles <= 0) return;   // uniform over the CTA

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::kStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < C::kNumAcc; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], C::kEpiWarps);
    }
    mbar_init(b_full, 1);
    mbar_init(mma_done, 1);
    *s_abort = 0;
    fence_mbar_init();
  }
  uint32_t* sHist = reinterpret_cast<uint32_t*>(smem + C::kHistOff);
  if constexpr (NTOK == 1) {
    for (int i = threadIdx.x; i < 4096; i += blockDim.x) sHist[i] = 0;
  } else {
    if constexpr (kRowHist) {
      uint4* h4 = reinterpret_cast<uint4*>(sHist);
      for (int i = threadIdx.x; i < NTOK * C::kRowHistWords / 4; i += blockDim.x)
        h4[i] = make_uint4(0u, 0u, 0u, 0u);
    }
  }

  // weights of the tile's tokens, widened to fp32
  for (int i = threadIdx.x; i < NTOK * kIdxHeads; i += blockDim.x) {
    const int tok = i / kIdxHeads;
    float wv = 0.f;
    if (tok < wk.ntok) {
      const int64_t row = static_cast<int64_t>(wk.b_row0) + i;   // b_row0 = token*16
      wv = __bfloat162float(args.w[row]);
    }
    sW[i] = wv;
  }
  if (warp == 1) {
    tmem_alloc(s_tmem, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      prefetch_tmap(&tmap_kbar);
      prefetch_tmap(&tmap_qidx);
      mbar_arrive_expect_tx(b_full, C::kBBytes);
      tma_load_2d(sB, &tmap_qidx, 0, wk.b_row0, b_full);
      int issued = 0;
      // row of M-tile m's first compressed key; paged caches look the page up (an M-tile of
      // 128 blocks lies inside one page), one tile ahead of its copy
      auto tile_row = [&](int m) -> int64_t {
        if constexpr (NTOK == 1) {
          if (args.pg.table != nullptr) {
            const int64_t r = pool_block(args.pg, wk.seq, 128ll * m);
            if (r < 0) report_error(args.st, kErrDevice, 204);
            return r < 0 ? static_cast<int64_t>(args.kbar_oob_row) : r;
          }
        }
        return wk.a_row0 + 128ll * m;
      };
      const uint64_t pol_stream = l2_policy_evict_first();
      int64_t row_next = wk.n_mtiles > 0 ? tile_row(wk.mt0) : 0;
      for (int i = 0; i < wk.n_mtiles; ++i) {
        const int s = i % C::kStages;
        const int64_t row = row_next;
        if (i + 1 < wk.n_mtiles) row_next = tile_row(wk.mt0 + i + 1);
        if (!mbar_wait(&empty[s], ((i / C::kStages) & 1) ^ 1, s_abort, args.st, 10)) break;
        mbar_arrive_expect_tx(&full[s], C::kABytes);
        if constexpr (NTOK == 1) {
          // decode: the compressed keys are read once per step; keep the scores (written
          // next, read back by the top-k) in L2 instead
          tma_load_2d_hint(sA + s * C::kABytes, &tmap_kbar, 0, static_cast<int32_t>(row),
                           &full[s], pol_stream);
        } else {
          tma_load_2d(sA + s * C::kABytes, &tmap_kbar, 0, static_cast<int32_t>(row), &full[s]);
        }
        ++issued;
      }
      if (*s_abort) {
        // let copies already in flight land before the CTA exits
        const int from = issued > C::kStages ? issued - C::kStages : 0;
        for (int j = from; j < issued; ++j) mbar_drain(&full[j % C::kStages], (j / C::kStages) & 1);
        mbar_drain(b_full, 0);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      bool ok = mbar_wait(b_full, 0, s_abort, args.st, 11);
      const uint32_t sA0 = smem_u32(sA), sB0 = smem_u32(sB);
      for (int i = 0; ok && i < wk.n_mtiles; ++i) {
        const int s = i % C::kStages;
        const int a = i % C::kNumAcc;
        if (!mbar_wait(&full[s], (i / C::kStages) & 1, s_abort, args.st, 12)) break;
        if (!mbar_wait(&acc_empty[a], ((i / C::kNumAcc) & 1) ^ 1, s_abort, args.st, 13)) break;
        tc_fence_after();
        const uint32_t d = tmem + a * C::kAccCols;
#pragma unroll
        for (int k = 0; k < kIdxDim / 16; ++k) {
          const uint64_t da = smem_desc_sw128(sA0 + s * C::kABytes + 32 * k, 0, 1024);
          const uint64_t db = smem_desc_sw128(sB0 + 32 * k, 0, 1024);
          umma_ss(d, da, db, C::kIdesc, k > 0 ? 1u : 0u);
        }
        umma_commit(&empty[s]);
        umma_commit(&acc_full[a]);
      }
      umma_commit(mma_done);
      mbar_drain(mma_done, 0);
    }
  } else {
    // ---------------- epilogue ----------------
    const int ew = warp - 2;
    const int quarter = warp & 3;          // TMEM lanes this warp may access
    const int part = ew / 4;               // which group of four tokens (prefill)
    constexpr int kTokPerWarp = NTOK == 16 ? 4 : 1;
    const int tok_base = part * kTokPerWarp;
    const uint64_t pol_keep = NTOK == 1 ? l2_policy_evict_last() : 0ull;
    for (int i = 0; i < wk.n_mtiles; ++i) {
      const int a = i % C::kNumAcc;
      const bool got = mbar_wait(&acc_full[a], (i / C::kNumAcc) & 1, s_abort, args.st, 14);
      if (__any_sync(0xffffffffu, !got)) break;   // also reconverges the warp
      tc_fence_after();
      const uint32_t tbase = tmem + (static_cast<uint32_t>(quarter * 32) << 16) + a * C::kAccCols +
                             tok_base * kIdxHeads;
      float sc[kTokPerWarp];
      if constexpr (NTOK == 16) {
        // two TMEM reads of two tokens each: the second is in flight while the first pair is
        // summed, and the accumulator is released once both have landed
        static_assert(kTokPerWarp == 4, "two pairs of tokens per warp");
        uint32_t acc0[32], acc1[32];
        tmem_ld32(tbase, acc0);
        tmem_wait_ld();
        reg_fence32(acc0);
        tmem_ld32(tbase + 32, acc1);
        sc[0] = head_weighted_relu_sum(acc0, sW + tok_base * kIdxHeads);
        sc[1] = head_weighted_relu_sum(acc0 + kIdxHeads, sW + (tok_base + 1) * kIdxHeads);
        tmem_wait_ld();
        reg_fence32(acc1);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_empty[a]);
        sc[2] = head_weighted_relu_sum(acc1, sW + (tok_base + 2) * kIdxHeads);
        sc[3] = head_weighted_relu_sum(acc1 + kIdxHeads, sW + (tok_base + 3) * kIdxHeads);
      } else {
        uint32_t acc[kIdxHeads];
        tmem_ld16(tbase, acc);
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_empty[a]);
        sc[0] = head_weighted_relu_sum(acc, sW + tok_base * kIdxHeads);
      }
      const int blk = 128 * (wk.mt0 + i) + quarter * 32 + lane;
#pragma unroll
      for (int j = 0; j < kTokPerWarp; ++j) {
        const int tok = tok_base + j;
        const float s = sc[j];
        const int pos = wk.pos0 + tok;
        const bool valid = tok < wk.ntok && blk < (NTOK == 1 ? wk.n_c : pos / kBlock);
        if (valid) {
          float* dst = args.scores + (wk.out_row0 + tok) * args.ld + blk;
          if constexpr (NTOK == 1) {
            st_global_hint(dst, s, pol_keep);
          } else {
            *dst = s;
            if constexpr (kRowHist) {   // this row's first-digit histogram (16-bit counters)
              const uint32_t bin = float_key(s) >> 20;
              atomicAdd(&sHist[tok * C::kRowHistWords + (bin >> 1)], 1u << ((bin & 1u) << 4));
            }
          }
        }
        if constexpr (NTOK == 1) {
          if (args.hist && valid) atomicAdd(&sHist[float_key(s) >> 20], 1u);
        }
      }
    }
  }
  __syncthreads();
  if constexpr (NTOK == 1) {
    if (args.hist) {
      uint32_t* dst = args.hist + static_cast<int64_t>(wk.out_row0) * 4096;
      for (int i = threadIdx.x; i < 4096; i += blockDim.x)
        if (sHist[i]) atomicAdd(&dst[i], sHist[i]);
    }
  } else {
    // select_mode 1: one warp per token row with more candidates than the budget finds the
    // row's threshold bin (the one the top-k's first pass would find): lane l sums bins
    // 4095 - 128 l down to 3968 - 128 l, a warp scan from the top finds the lane whose range
    // holds the topk-th key, and that lane walks its bins
    if (kRowHist && !*s_abort && warp < NTOK) {
      const int tok = warp;
      const int n = (wk.pos0 + tok) / kBlock;
      if (tok < wk.ntok && n > args.topk) {   // uniform over the warp
        const uint32_t* h = sHist + tok * C::kRowHistWords;
        const int top = 4095 - 128 * lane;   // this lane's bins: top .. top - 127
        int local = 0;
#pragma unroll 8
        for (int wd = 0; wd < 64; ++wd) {
          const uint32_t v = h[(top >> 1) - wd];
          local += static_cast<int>((v & 0xffffu) + (v >> 16));
        }
        int incl = local;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int y = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += y;
        }
        int running = incl - local;   // keys in the bins above this lane's range
        if (running < args.topk && incl >= args.topk) {
          for (int bin = top; bin > top - 128; --bin) {
            const uint32_t v = h[bin >> 1];
            const int c = static_cast<int>((bin & 1) ? (v >> 16) : (v & 0xffffu));
            if (running + c >= args.topk) {
              int32_t* ri = args.rinfo + (wk.out_row0 + tok) * 4;
              ri[0] = bin;
              ri[1] = running;
              ri[2] = c;
              ri[3] = n;
              break;
            }
            running += c;
          }
        }
      }
    }
  }
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

}  // namespace qsa
