// qsa_misc.cuh -- bandwidth-bound QSA kernels: sequence metadata, block compression,
// cache append, radix top-k, the attention union plan and the decode split combine.
#pragma once

#include "qsa_common.cuh"

namespace qsa {

// Per-sequence metadata derived on the device from cu_seqlens.
struct SeqMeta {
  int64_t tok0;      // first token of the sequence in the packed arrays
  int64_t kbar0;     // first compressed block of the sequence in the packed kbar array
  int32_t len;       // tokens
  int32_t score_tile0;  // first 16-token score tile (global numbering)
  int32_t attn_tile0;   // first attention tile (rows_per_tile tokens each)
  int32_t pad;
};

// Warp-wide exclusive scan of one int per lane; *total receives the warp sum.
__device__ __forceinline__ int warp_count_scan(int v, int* total) {
  const int lane = threadIdx.x & 31;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  *total = __shfl_sync(0xffffffffu, x, 31);
  return x - v;
}

// ---------------------------------------------------------------------------------------
// Block-wide exclusive scan of one int per thread (blockDim.x a multiple of 32, <= 1024).
__device__ __forceinline__ int block_excl_scan(int v, int* sh /*[33]*/, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nw = (blockDim.x + 31) >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) sh[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int y = lane < nw ? sh[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int z = __shfl_up_sync(0xffffffffu, y, o);
      if (lane >= o) y += z;
    }
    sh[lane] = y;   // inclusive prefix of warp totals
  }
  __syncthreads();
  int excl = x - v + (warp > 0 ? sh[warp - 1] : 0);
  *total = sh[nw - 1];
  __syncthreads();
  return excl;
}

// The same scan with one barrier: every warp reads all warp totals and scans them itself.
// sh[0 .. warps) is written before the barrier and read after it, so the caller must pass at
// least one more __syncthreads before sh is written again (the next call included).
__device__ __forceinline__ int block_excl_scan_1bar(int v, int* sh /*[32]*/, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nw = (blockDim.x + 31) >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) sh[warp] = x;
  __syncthreads();
  int t = lane < nw ? sh[lane] : 0;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, t, o);
    if (lane >= o) t += y;
  }
  const int before = __shfl_sync(0xffffffffu, t, (warp + 31) & 31);   // inclusive, warp - 1
  *total = __shfl_sync(0xffffffffu, t, nw - 1);
  return x - v + (warp > 0 ? before : 0);
}

// One CTA: metadata for every sequence (prefix sums over blocks and tiles).
__global__ void __launch_bounds__(1024) k_seq_meta(const int32_t* __restrict__ cu, int num_seqs,
                                                   int rows_per_tile, SeqMeta* __restrict__ meta,
                                                   DevStatus st) {
  __shared__ int sh[33];
  int64_t carry_blk = 0;
  int carry_st = 0, carry_at = 0;
  for (int base = 0; base < num_seqs; base += blockDim.x) {
    const int s = base + threadIdx.x;
    int L = 0;
    int64_t t0 = 0;
    if (s < num_seqs) {
      t0 = cu[s];
      L = cu[s + 1] - cu[s];
      if (L < 0) {
        report_error(st, kErrDevice, 100);
        L = 0;
      }
    }
    const int nb = L / kBlock, nst = (L + 15) / 16,
              nat = rows_per_tile > 0 ? (L + rows_per_tile - 1) / rows_per_tile : 0;
    int tot_b, tot_s, tot_a;
    const int eb = block_excl_scan(nb, sh, &tot_b);
    const int es = block_excl_scan(nst, sh, &tot_s);
    const int ea = block_excl_scan(nat, sh, &tot_a);
    if (s < num_seqs) {
      SeqMeta m;
      m.tok0 = t0;
      m.kbar0 = carry_blk + eb;
      m.len = L;
      m.score_tile0 = carry_st + es;
      m.attn_tile0 = carry_at + ea;
      m.pad = 0;
      meta[s] = m;
    }
    carry_blk += tot_b;
    carry_st += tot_s;
    carry_at += tot_a;
  }
  if (threadIdx.x == 0) {   // sentinel entry: totals
    SeqMeta m;
    m.tok0 = 0;
    m.kbar0 = carry_blk;
    m.len = 0;
    m.score_tile0 = carry_st;
    m.attn_tile0 = carry_at;
    m.pad = 0;
    meta[num_seqs] = m;
  }
}

// Sequence owning global tile `gt` (tile0 of meta is non-decreasing; meta[num_seqs] holds totals).
template <bool kAttnTiles>
__device__ __forceinline__ int find_seq_of_tile(const SeqMeta* meta, int num_seqs, int gt) {
  int lo = 0, hi = num_seqs - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    const int t0 = kAttnTiles ? meta[mid].attn_tile0 : meta[mid].score_tile0;
    if (t0 <= gt) lo = mid; else hi = mid - 1;
  }
  return lo;
}

__device__ __forceinline__ int find_seq_of_token(const SeqMeta* meta, int num_seqs, int64_t t) {
  int lo = 0, hi = num_seqs - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (meta[mid].tok0 <= t) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// n_c (number of candidate blocks) of every token row: floor(pos / 4).
__global__ void k_row_nc(const SeqMeta* __restrict__ meta, int num_seqs, int64_t total,
                         int32_t* __restrict__ n_c) {
  for (int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; t < total;
       t += (int64_t)gridDim.x * blockDim.x) {
    const int s = find_seq_of_token(meta, num_seqs, t);
    n_c[t] = static_cast<int32_t>((t - meta[s].tok0) / kBlock);
  }
}

// ---------------------------------------------------------------------------------------
// Step a1, fixed order: kbar = bf16_rne(((k0 + k1) + k2) + k3) * 0.25) with fp32 sums.
// One thread per (block, 8-dim slice): four 16-byte loads, one 16-byte store.
__device__ __forceinline__ uint4 compress4(uint4 a, uint4 b, uint4 c, uint4 d) {
  const uint32_t* pa = reinterpret_cast<const uint32_t*>(&a);
  const uint32_t* pb = reinterpret_cast<const uint32_t*>(&b);
  const uint32_t* pc = reinterpret_cast<const uint32_t*>(&c);
  const uint32_t* pd = reinterpret_cast<const uint32_t*>(&d);
  uint4 out;
  uint32_t* po = reinterpret_cast<uint32_t*>(&out);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float lo = __uint_as_float(pa[i] << 16), hi = __uint_as_float(pa[i] & 0xffff0000u);
    lo = __fadd_rn(lo, __uint_as_float(pb[i] << 16));
    hi = __fadd_rn(hi, __uint_as_float(pb[i] & 0xffff0000u));
    lo = __fadd_rn(lo, __uint_as_float(pc[i] << 16));
    hi = __fadd_rn(hi, __uint_as_float(pc[i] & 0xffff0000u));
    lo = __fadd_rn(lo, __uint_as_float(pd[i] << 16));
    hi = __fadd_rn(hi, __uint_as_float(pd[i] & 0xffff0000u));
    po[i] = pack_bf16x2(__fmul_rn(lo, 0.25f), __fmul_rn(hi, 0.25f));
  }
  return out;
}

__global__ void k_compress(const uint4* __restrict__ k_idx, const SeqMeta* __restrict__ meta,
                           int num_seqs, uint4* __restrict__ kbar) {
  const int64_t total_blocks = meta[num_seqs].kbar0;
  const int64_t n = total_blocks * 8;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t gb = i >> 3;
    const int part = static_cast<int>(i & 7);
    // sequence of packed block gb: last s with kbar0 <= gb
    int lo = 0, hi = num_seqs - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (meta[mid].kbar0 <= gb) lo = mid; else hi = mid - 1;
    }
    const int64_t b = gb - meta[lo].kbar0;
    const int64_t tok = meta[lo].tok0 + 4 * b;
    const uint4* src = k_idx + tok * 8 + part;
    kbar[gb * 8 + part] = compress4(src[0], src[8], src[16], src[24]);
  }
}

// ---------------------------------------------------------------------------------------
// Step a5: append.  Part 1 copies K/V rows into the blocked cache and (re)computes the
// compressed keys of the blocks the new tokens touch.  The first touched block may hold
// older tokens whose running sum is in kbar_partial; the last touched block may stay
// incomplete and leaves its sum there.  The same thread handles both ends of a sequence
// so that the read of the old partial precedes the write of the new one.
struct AppendParams {
  const uint4* k;      // [B][n_new][2][128] bf16 as 16-byte units
  const uint4* v;
  const uint4* k_idx;  // [B][n_new][64]
  const int32_t* counts;  // [B] or null
  int32_t n_new;
  int32_t batch;
  int32_t capacity;
  uint4* k_blocks;     // [pool pages][2][page blocks][4][128] (contiguous: [B][2][cap/4][4][128])
  uint4* v_blocks;
  uint4* kbar;         // [pool pages][page blocks][64] (contiguous: [B][cap/4][64])
  float* partial;      // [B][64]
  const int32_t* len;  // [B]
  Paging pg;
  DevStatus st;
};

__device__ __forceinline__ int append_count(const AppendParams& p, int b) {
  int c = p.counts ? p.counts[b] : p.n_new;
  return c < 0 ? 0 : (c > p.n_new ? p.n_new : c);
}

// Copies: one work item per 16 bytes of K and V (items 0 .. batch * n_new * 32).
__device__ __forceinline__ void append_copy_item(const AppendParams& p, int64_t i) {
  const int64_t per_tok = 2 * 16;                       // 2 heads x 16 units of 16 B
  {
    const int b = static_cast<int>(i / (static_cast<int64_t>(p.n_new) * per_tok));
    const int64_t rem = i - static_cast<int64_t>(b) * p.n_new * per_tok;
    const int j = static_cast<int>(rem / per_tok);
    const int g = static_cast<int>((rem / 16) & 1);
    const int u = static_cast<int>(rem & 15);
    if (j >= append_count(p, b)) return;
    const int64_t pos = static_cast<int64_t>(p.len[b]) + j;
    if (pos >= p.capacity) {
      report_error(p.st, kErrDevice, 200);
      return;
    }
    const int64_t row0 = pool_kv_row(p.pg, b, g, pos / 4);   // the block's first row
    if (row0 < 0) {
      report_error(p.st, kErrDevice, 202);
      return;
    }
    const int64_t dst = (row0 + pos % 4) * 16 + u;
    const int64_t src = ((static_cast<int64_t>(b) * p.n_new + j) * 2 + g) * 16 + u;
    p.k_blocks[dst] = p.k[src];
    p.v_blocks[dst] = p.v[src];
    // The last appended token of a sequence zeroes the rest of its block, so that rows not
    // yet written are finite (attention reads whole blocks and masks the future rows).
    if (j == append_count(p, b) - 1) {
      for (int64_t q = pos + 1; q < (pos / 4) * 4 + 4; ++q) {
        const int64_t dz = (row0 + q % 4) * 16 + u;
        p.k_blocks[dz] = make_uint4(0, 0, 0, 0);
        p.v_blocks[dz] = make_uint4(0, 0, 0, 0);
      }
    }
  }
}

// Compressed keys: one work item per (sequence, touched block, 8-dim slice), items 0 ..
// batch * max_blocks_touched * 8.  Slot 0 of each sequence handles the first and the last
// touched block; slots 1.. the complete middle ones.
__device__ __forceinline__ void append_kbar_item(const AppendParams& p, int64_t i,
                                                 int max_blocks_touched) {
  const int64_t slots = static_cast<int64_t>(max_blocks_touched);
  {
    const int b = static_cast<int>(i / (slots * 8));
    const int64_t slot = (i / 8) % slots;
    const int part = static_cast<int>(i & 7);
    const int cnt = append_count(p, b);
    if (cnt == 0) return;
    const int64_t L0 = p.len[b];
    const int64_t L1 = L0 + cnt;
    if (L1 > p.capacity) {
      if (slot == 0 && part == 0) report_error(p.st, kErrDevice, 201);
      return;
    }
    const int64_t jf = L0 / 4, jl = (L1 - 1) / 4;
    const uint4* kin = p.k_idx + static_cast<int64_t>(b) * p.n_new * 8 + part;  // token j at +8j
    float* part_sum = p.partial + static_cast<int64_t>(b) * 64 + part * 8;
    uint4* kb_out = p.kbar + part;   // + 8 x the pool block
    auto add_tokens = [&](float* acc, int64_t from, int64_t to, bool start_from_first) {
      // sum tokens [from, to) (absolute positions) into acc in order
      for (int64_t pos = from; pos < to; ++pos) {
        const uint4 x = kin[(pos - L0) * 8];
        const uint32_t* px = reinterpret_cast<const uint32_t*>(&x);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float lo = __uint_as_float(px[q] << 16), hi = __uint_as_float(px[q] & 0xffff0000u);
          if (start_from_first && pos == from) {
            acc[2 * q] = lo;
            acc[2 * q + 1] = hi;
          } else {
            acc[2 * q] = __fadd_rn(acc[2 * q], lo);
            acc[2 * q + 1] = __fadd_rn(acc[2 * q + 1], hi);
          }
        }
      }
    };
    auto finish = [&](const float* acc, int64_t j, bool complete) {
      if (complete) {
        uint4 o;
        uint32_t* po = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
        for (int q = 0; q < 4; ++q)
          po[q] = pack_bf16x2(__fmul_rn(acc[2 * q], 0.25f), __fmul_rn(acc[2 * q + 1], 0.25f));
        const int64_t pb = pool_block(p.pg, b, j);
        if (pb < 0) {
          report_error(p.st, kErrDevice, 203);
          return;
        }
        kb_out[pb * 8] = o;
      } else {
#pragma unroll
        for (int q = 0; q < 8; ++q) part_sum[q] = acc[q];
      }
    };
    float acc[8];
    if (slot == 0) {
      // first touched block
      const int64_t end_f = (4 * jf + 4 < L1) ? 4 * jf + 4 : L1;
      if (L0 % 4 != 0) {
#pragma unroll
        for (int q = 0; q < 8; ++q) acc[q] = part_sum[q];
        add_tokens(acc, L0, end_f, false);
      } else {
        add_tokens(acc, L0, end_f, true);
      }
      finish(acc, jf, end_f == 4 * jf + 4);
      if (jl != jf) {   // last touched block starts fresh
        add_tokens(acc, 4 * jl, L1, true);
        finish(acc, jl, L1 == 4 * jl + 4);
      }
    } else {
      const int64_t j = jf + slot;       // middle blocks jf+1 .. jl-1 are complete and new
      if (j >= jl) return;
      add_tokens(acc, 4 * j, 4 * j + 4, true);
      finish(acc, j, true);
    }
  }
}

// K/V copies and compressed-key updates in one launch (both read the lengths before the
// append); k_append_len then advances the lengths.
__global__ void k_append(AppendParams p, int max_blocks_touched) {
  pdl_trigger();
  pdl_wait();   // launched as a programmatic dependent of the caller's last kernel
  const int64_t n_copy = static_cast<int64_t>(p.batch) * p.n_new * 32;
  const int64_t n_kbar = static_cast<int64_t>(p.batch) * max_blocks_touched * 8;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n_copy + n_kbar;
       i += (int64_t)gridDim.x * blockDim.x) {
    if (i < n_copy) append_copy_item(p, i);
    else append_kbar_item(p, i - n_copy, max_blocks_touched);
  }
}

// Zeroes n 32-bit words (the decode histograms and candidate counters).
__global__ void k_zero_words(uint32_t* __restrict__ p, int64_t n) {
  pdl_trigger();
  pdl_wait();
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x)
    p[i] = 0u;
}

__global__ void k_append_len(int32_t* len, const int32_t* counts, int32_t n_new, int batch) {
  pdl_trigger();
  pdl_wait();   // every k_append thread has read len
  for (int b = blockIdx.x * blockDim.x + threadIdx.x; b < batch; b += gridDim.x * blockDim.x) {
    int c = counts ? counts[b] : n_new;
    c = c < 0 ? 0 : (c > n_new ? n_new : c);
    len[b] += c;
  }
}

// Attention plan.  A tile is up to R consecutive query tokens of one sequence (R = 1 for
// decode, whose records the decode top-k writes directly).  The tile's key set is the union U
// of its tokens' selected blocks and their own blocks, in ascending block order.  For every token r and every 32-block chunk q of the
// union, mask[r][q] has bit u set when union block 32q+u is selected by r or is r's own
// block; tail[r] is the union position of r's own block.
struct PlanLayout {
  int32_t R;         // tokens per tile
  int32_t umax;      // union capacity per tile (multiple of 32)
  int64_t stride;    // int32 entries per tile record
  // record: [0] = U, [1] = number of tokens, [2] = position of token 0 in its sequence,
  //         [3] unused, [4..4+R) = union position of each token's own block,
  //         [4+R .. 4+R+umax) = union block ids, then R * (umax/32) mask words
  __host__ __device__ int64_t tail_off() const { return 4; }
  __host__ __device__ int64_t union_off() const { return 4 + R; }
  __host__ __device__ int64_t mask_off() const { return 4 + R + umax; }
};

__host__ __device__ inline PlanLayout make_plan_layout(int R, int topk) {
  PlanLayout pl;
  pl.R = R;
  pl.umax = ((R * (topk + 1)) + 31) / 32 * 32;
  pl.stride = 4 + R + pl.umax + static_cast<int64_t>(R) * (pl.umax / 32);
  pl.stride = (pl.stride + 3) / 4 * 4;   // 16-byte aligned records
  return pl;
}

// Decode: the plan record of a one-token tile, written straight from the token's selection
// sel[0 .. k) (ascending, all below its own block c): the union is the selection followed by
// c, every union block is attended, and c sits at union position k.  Called by all threads of
// a CTA after sel is complete.
__device__ __forceinline__ void write_decode_plan(int32_t* rec, const PlanLayout& pl,
                                                  const int32_t* sel, int k, int c, int p) {
  const int U = k + 1;
  int32_t* uni = rec + pl.union_off();
  for (int j = threadIdx.x; j < k; j += blockDim.x) uni[j] = sel[j];
  uint32_t* m = reinterpret_cast<uint32_t*>(rec + pl.mask_off());
  const int nq = (U + 31) / 32;
  for (int q = threadIdx.x; q < nq; q += blockDim.x) {
    const int rem = U - 32 * q;
    m[q] = rem >= 32 ? 0xffffffffu : ((1u << rem) - 1u);
  }
  if (threadIdx.x == 0) {
    uni[k] = c;
    rec[0] = U;
    rec[1] = 1;
    rec[2] = p;
    rec[pl.tail_off()] = k;
  }
}

// ---------------------------------------------------------------------------------------
// Step a3: top-k per row by radix select on order-preserving uint32 keys, with the selected
// blocks emitted in ascending index order and ties at the threshold broken toward lower
// indices.  One 512-thread CTA works on a row.  The kernels (k_topk for score rows; the
// collect/finish pair for decode) narrow a row to the candidates at or above the threshold bin
// of the first digit (key bits 31..20) and finish there; topk_row, the full-row select with
// digits of 12, 12 and 8 bits and an ordered compaction over the whole row, serves rows whose
// candidates overflow.  It takes the first-digit histogram ready-made when one is given.
constexpr int kTopkThreads = 512;
constexpr int kTopkWarps = kTopkThreads / 32;
constexpr int kTopkBins = 4096;

struct TopkShared {
  uint32_t hist[kTopkBins];
  uint32_t hist3[256];   // third digit of the candidate select, cleared with the second's
  int sh[40];
  int sel[4];   // threshold bin, keys above it, keys in it
  int wgt[kTopkWarps];
  int weq[kTopkWarps];
};
// Byte offset of the cached score row in k_topk's dynamic shared memory (16-byte aligned for
// the float4 copy; the host sizes the allocation with the same constant).
constexpr int kTopkSharedBytes = (static_cast<int>(sizeof(TopkShared)) + 127) / 128 * 128;

// Find the bin of `hist` where the count of keys in higher bins first reaches `need` (bins
// scanned from the top).  Returns the bin; *above receives the count of keys in higher bins and
// *in_bin (if given) the bin's own count.  nbins is kTopkBins (eight bins a thread, read as
// two uint4, thread 0 holding the highest) or at most kTopkThreads (one bin a thread).  One
// block scan places every thread's bins; only the thread whose range holds the crossing walks
// its bins.  Two barriers; the histogram may be rewritten as soon as this returns.
static_assert(kTopkBins == 8 * kTopkThreads, "topk_find_bin holds eight bins a thread");
__device__ __forceinline__ int topk_find_bin(TopkShared& S, const uint32_t* hist, int nbins,
                                             int need, int* above, int* in_bin = nullptr) {
  const int tid = threadIdx.x;
  int tot;
  if (nbins == kTopkBins) {
    const int lo = kTopkBins - 8 * (tid + 1);
    const uint4 h0 = *reinterpret_cast<const uint4*>(hist + lo);
    const uint4 h1 = *reinterpret_cast<const uint4*>(hist + lo + 4);
    const int v[8] = {static_cast<int>(h0.x), static_cast<int>(h0.y), static_cast<int>(h0.z),
                      static_cast<int>(h0.w), static_cast<int>(h1.x), static_cast<int>(h1.y),
                      static_cast<int>(h1.z), static_cast<int>(h1.w)};
    int local = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) local += v[j];
    int running = block_excl_scan_1bar(local, S.sh, &tot);   // keys in bins above my range
    if (running < need && running + local >= need) {
#pragma unroll
      for (int j = 7; j >= 0; --j) {
        if (running < need && running + v[j] >= need) {
          S.sel[0] = lo + j;
          S.sel[1] = running;
          S.sel[2] = v[j];
        }
        running += v[j];
      }
    }
  } else {
    const int bin = nbins - 1 - tid;
    const int c = bin >= 0 ? static_cast<int>(hist[bin]) : 0;
    const int running = block_excl_scan_1bar(c, S.sh, &tot);
    if (bin >= 0 && running < need && running + c >= need) {
      S.sel[0] = bin;
      S.sel[1] = running;
      S.sel[2] = c;
    }
  }
  __syncthreads();
  *above = S.sel[1];
  if (in_bin) *in_bin = S.sel[2];
  return S.sel[0];
}

// Zero the first nbins words of a histogram (nbins a multiple of 4, the array 16-byte aligned).
__device__ __forceinline__ void clear_bins(uint32_t* h, int nbins) {
  for (int i = threadIdx.x; i < nbins / 4; i += blockDim.x)
    reinterpret_cast<uint4*>(h)[i] = make_uint4(0u, 0u, 0u, 0u);
}

__device__ __forceinline__ void topk_row(const float* __restrict__ src, int n, int topk,
                                         const uint32_t* hist1, int32_t* __restrict__ out,
                                         TopkShared& S) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int need = topk;
  // ---- digit 1: key bits [31:20] ----
  if (hist1) {
    for (int i = tid; i < kTopkBins; i += kTopkThreads) S.hist[i] = hist1[i];
  } else {
    clear_bins(S.hist, kTopkBins);
    __syncthreads();
    for (int base = 0; base < n; base += kTopkThreads) {
      const int i = base + tid;
      const uint32_t bin = i < n ? (float_key(src[i]) >> 20) : 0xffffffffu;
      const unsigned act = __ballot_sync(0xffffffffu, i < n);
      if (i < n) {
        const unsigned peers = __match_any_sync(act, bin);   // lanes sharing this bin
        if (lane == __ffs(peers) - 1) atomicAdd(&S.hist[bin], static_cast<uint32_t>(__popc(peers)));
      }
    }
  }
  __syncthreads();
  int above;
  const uint32_t b1 = static_cast<uint32_t>(topk_find_bin(S, S.hist, kTopkBins, need, &above));
  need -= above;
  // ---- digit 2: bits [19:8] among keys in bin b1 ----
  clear_bins(S.hist, kTopkBins);
  __syncthreads();
  for (int i = tid; i < n; i += kTopkThreads) {
    const uint32_t key = float_key(src[i]);
    if ((key >> 20) == b1) atomicAdd(&S.hist[(key >> 8) & 0xfffu], 1u);
  }
  __syncthreads();
  const uint32_t b2 = static_cast<uint32_t>(topk_find_bin(S, S.hist, kTopkBins, need, &above));
  need -= above;
  // ---- digit 3: bits [7:0] ----
  const uint32_t pre = (b1 << 12) | b2;
  clear_bins(S.hist, 256);
  __syncthreads();
  for (int i = tid; i < n; i += kTopkThreads) {
    const uint32_t key = float_key(src[i]);
    if ((key >> 8) == pre) atomicAdd(&S.hist[key & 0xffu], 1u);
  }
  __syncthreads();
  const uint32_t b3 = static_cast<uint32_t>(topk_find_bin(S, S.hist, 256, need, &above));
  need -= above;
  const uint32_t T = (pre << 8) | b3;   // the k-th largest key
  const int need_eq = need;             // keys equal to T to take, lowest indices first
  // ---- ordered output: each warp owns a contiguous segment ----
  const int seg = ((n + kTopkWarps - 1) / kTopkWarps + 31) / 32 * 32;
  const int s0 = warp * seg;
  const int s1 = min(n, s0 + seg);
  int c_gt = 0, c_eq = 0;
  for (int base = s0; base < s1; base += 32) {
    const int i = base + lane;
    const uint32_t key = i < s1 ? float_key(src[i]) : 0u;
    c_gt += __popc(__ballot_sync(0xffffffffu, i < s1 && key > T));
    c_eq += __popc(__ballot_sync(0xffffffffu, i < s1 && key == T));
  }
  if (lane == 0) {
    S.wgt[warp] = c_gt;
    S.weq[warp] = c_eq;
  }
  __syncthreads();
  int eq_before = 0, out_before = 0;
  for (int w = 0; w < warp; ++w) {
    const int eqw = S.weq[w];
    const int takew = min(max(need_eq - eq_before, 0), eqw);
    out_before += S.wgt[w] + takew;
    eq_before += eqw;
  }
  const unsigned lt_mask = (1u << lane) - 1u;
  for (int base = s0; base < s1; base += 32) {
    const int i = base + lane;
    const uint32_t key = i < s1 ? float_key(src[i]) : 0u;
    const bool gt = i < s1 && key > T;
    const bool eq = i < s1 && key == T;
    const unsigned eqm = __ballot_sync(0xffffffffu, eq);
    const int eq_rank = eq_before + __popc(eqm & lt_mask);
    const bool take = gt || (eq && eq_rank < need_eq);
    const unsigned tm = __ballot_sync(0xffffffffu, take);
    if (take) {
      const int pos = out_before + __popc(tm & lt_mask);
      if (pos < topk) out[pos] = i;
    }
    out_before += __popc(tm);
    eq_before += __popc(eqm);
  }
  __syncthreads();
}


// ---------------------------------------------------------------------------------------
// Long rows (decode): top-k from a first-digit histogram built while scoring, in two steps.
//   k_topk_collect  (rows x parts CTAs): every CTA finds the threshold bin B1 of its row from
//                   the histogram and appends (key, index) of each score in bins >= B1 to the
//                   row's candidate list (at most topk - 1 + hist[B1] entries); the row's first
//                   CTA also records B1 and the counts above and in it (row info).
//   k_topk_finish   (one CTA per row): exact radix select among the candidates (digits 2, 3),
//                   then the ascending index list through shared-memory bitmaps: every key
//                   above the threshold, plus the lowest-index keys equal to it.
// A row whose candidates would not fit `cap` is left to the full-row select (topk_row).
constexpr int kCandThreads = 512;
constexpr int kCandBins = 4096 / kCandThreads;   // histogram bins per thread
static_assert(kCandBins % 4 == 0, "hist_threshold_bin loads its bins as uint4");

// Threshold bin of a row from its 4096-bin histogram: thread t holds bins 4096-kCandBins(t+1)
// .. 4095-kCandBins t in registers (the highest bins go to thread 0).  Returns the bin where the
// count of keys in higher bins first reaches `topk`; *above receives that count and *in_bin the
// bin's own.
__device__ __forceinline__ int hist_threshold_bin(const uint32_t* __restrict__ h, int topk,
                                                  int* above_out, int* in_bin_out, int* sh /*[40]*/) {
  const int lo = 4096 - kCandBins * (static_cast<int>(threadIdx.x) + 1);
  const uint4* h4 = reinterpret_cast<const uint4*>(h + lo);
  uint32_t v[kCandBins];
#pragma unroll
  for (int q = 0; q < kCandBins / 4; ++q) {
    const uint4 x = h4[q];
    v[4 * q] = x.x;
    v[4 * q + 1] = x.y;
    v[4 * q + 2] = x.z;
    v[4 * q + 3] = x.w;
  }
  int local = 0;
#pragma unroll
  for (int j = 0; j < kCandBins; ++j) local += static_cast<int>(v[j]);
  int tot;
  int running = block_excl_scan_1bar(local, sh, &tot);   // keys in bins above this thread's range
#pragma unroll
  for (int j = kCandBins - 1; j >= 0; --j) {
    const int c = static_cast<int>(v[j]);
    if (running < topk && running + c >= topk) {
      sh[36] = lo + j;
      sh[37] = running;
      sh[38] = c;
    }
    running += c;
  }
  __syncthreads();
  const int bin = sh[36];
  *above_out = sh[37];
  *in_bin_out = sh[38];
  return bin;   // sh[36..38] is not written again in this CTA
}

// Each CTA covers `per` (a multiple of 4) scores of one row in passes of 64 scores a thread
// (usually one pass).  The first pass's loads go out before the threshold bin is looked up in
// the histogram, so that lookup hides under them; after the loads one block scan places the
// pass's candidates with a single atomic on the row's counter.  Few, large CTAs: a grid of
// small ones spent most of its time starting them.
constexpr int kCollectPerThread = 64;
constexpr int kCollectPerCta = kCandThreads * kCollectPerThread;   // one pass
__global__ void __launch_bounds__(kCandThreads, 1) k_topk_collect(
    const float* __restrict__ scores, int64_t ld, const int32_t* __restrict__ n_c, int topk,
    int parts, int cap, const uint32_t* __restrict__ hist, int32_t* __restrict__ cand_cnt,
    uint64_t* __restrict__ cand, int32_t* __restrict__ rinfo) {
  pdl_trigger();
  pdl_wait();
  __shared__ int sh[40];
  __shared__ int s_base;
  const int r = blockIdx.x / parts, part = blockIdx.x % parts;
  const int n = n_c[r];
  if (n <= topk) return;
  const int per = ((n + parts - 1) / parts + 3) & ~3;
  const int a = part * per, e = min(n, a + per);
  const float* src = scores + static_cast<int64_t>(r) * ld;
  uint64_t* out = cand + static_cast<int64_t>(r) * cap;
  uint32_t b1 = 0;
  for (int base = a; base < e; base += kCollectPerCta) {
    float x[kCollectPerThread];
#pragma unroll
    for (int q = 0; q < kCollectPerThread / 4; ++q) {
      const int i = base + 4 * (q * kCandThreads + static_cast<int>(threadIdx.x));
      float4 f = make_float4(0.f, 0.f, 0.f, 0.f);
      if (i < e) f = *reinterpret_cast<const float4*>(src + i);   // i % 4 == 0, row 16B-aligned
      x[4 * q] = f.x;
      x[4 * q + 1] = f.y;
      x[4 * q + 2] = f.z;
      x[4 * q + 3] = f.w;
    }
    if (base == a) {
      int above, in_b1;
      b1 = static_cast<uint32_t>(
          hist_threshold_bin(hist + static_cast<int64_t>(r) * 4096, topk, &above, &in_b1, sh));
      if (part == 0 && threadIdx.x == 0) {
        rinfo[4 * r] = static_cast<int32_t>(b1);
        rinfo[4 * r + 1] = above;
        rinfo[4 * r + 2] = in_b1;
      }
      if (above + in_b1 > cap) return;   // overflow: the finish kernel takes the full-row path
    }
    uint64_t take = 0;
#pragma unroll
    for (int j = 0; j < kCollectPerThread; ++j) {
      const int i = base + 4 * ((j / 4) * kCandThreads + static_cast<int>(threadIdx.x)) + (j & 3);
      if (i < e && (float_key(x[j]) >> 20) >= b1) take |= 1ull << j;
    }
    int tot;
    const int ex = block_excl_scan_1bar(__popcll(take), sh, &tot);
    if (tot == 0) {            // uniform: tot is the block total
      __syncthreads();         // the scan's totals are read before the next pass rewrites them
      continue;
    }
    if (threadIdx.x == 0) s_base = atomicAdd(cand_cnt + r, tot);
    __syncthreads();
    int slot = s_base + ex;
#pragma unroll
    for (int j = 0; j < kCollectPerThread; ++j) {
      if (take & (1ull << j)) {
        const int i = base + 4 * ((j / 4) * kCandThreads + static_cast<int>(threadIdx.x)) + (j & 3);
        if (slot < cap) out[slot] = (static_cast<uint64_t>(float_key(x[j])) << 32) | static_cast<uint32_t>(i);
        ++slot;
      }
    }
    __syncthreads();   // s_base is rewritten by the next pass
  }
}

// Exact top-k among candidates c[0 .. C) (composites key << 32 | block, in any order) that hold
// every key at or above the threshold bin b1 of the first digit; `need` is topk minus the keys
// in bins above b1.  Digits 2 (key bits 19..8) and 3 (bits 7..0) among the keys of bin b1 give
// the k-th largest key T; the selection is every key above T plus the need_eq lowest-index keys
// equal to T, emitted in ascending block order through two bitmaps of nwords words (sel, eqb)
// and prefix popcounts.  Called by all kTopkThreads threads of the CTA.
__device__ __forceinline__ void topk_select_candidates(TopkShared& S, const uint64_t* c, int C,
                                                       uint32_t b1, int need, uint32_t* sel,
                                                       uint32_t* eqb, int nwords, int topk,
                                                       int32_t* __restrict__ out) {
  const int tid = threadIdx.x;
  int above;
  clear_bins(S.hist, kTopkBins);
  clear_bins(S.hist3, 256);
  for (int i = tid; i < nwords; i += blockDim.x) {
    sel[i] = 0;
    eqb[i] = 0;
  }
  __syncthreads();
  for (int i = tid; i < C; i += blockDim.x) {
    const uint32_t key = static_cast<uint32_t>(c[i] >> 32);
    if ((key >> 20) == b1) atomicAdd(&S.hist[(key >> 8) & 0xfffu], 1u);
  }
  __syncthreads();
  const uint32_t b2 = static_cast<uint32_t>(topk_find_bin(S, S.hist, kTopkBins, need, &above));
  need -= above;
  const uint32_t pre = (b1 << 12) | b2;
  for (int i = tid; i < C; i += blockDim.x) {
    const uint32_t key = static_cast<uint32_t>(c[i] >> 32);
    if ((key >> 8) == pre) atomicAdd(&S.hist3[key & 0xffu], 1u);
  }
  __syncthreads();
  const uint32_t b3 = static_cast<uint32_t>(topk_find_bin(S, S.hist3, 256, need, &above));
  need -= above;
  const uint32_t T = (pre << 8) | b3;
  const int need_eq = need;
  // bitmaps: keys above T are selected; keys equal to T are marked in eqb
  for (int i = tid; i < C; i += blockDim.x) {
    const uint32_t key = static_cast<uint32_t>(c[i] >> 32);
    const uint32_t ix = static_cast<uint32_t>(c[i]);
    if (key > T) atomicOr(&sel[ix >> 5], 1u << (ix & 31));
    else if (key == T) atomicOr(&eqb[ix >> 5], 1u << (ix & 31));
  }
  __syncthreads();
  const int per = (nwords + kTopkThreads - 1) / kTopkThreads;
  const int w0 = tid * per, w1 = min(nwords, w0 + per);
  // One block scan places everything: fewer than topk (<= 1024) keys lie above T, so a
  // thread's count of them fits 11 bits, under its count of keys equal to T.  The need_eq
  // lowest-index equal keys join the selection, which is emitted in ascending block order.
  {
    int l_gt = 0, l_eq = 0;
    for (int w = w0; w < w1; ++w) {
      l_gt += __popc(sel[w]);
      l_eq += __popc(eqb[w]);
    }
    int tot;
    const int ex = block_excl_scan_1bar(l_eq * 2048 + l_gt, S.sh, &tot);
    const int eq_before = ex >> 11, gt_before = ex & 2047;
    int take = min(max(need_eq - eq_before, 0), l_eq);
    int pos = gt_before + min(eq_before, need_eq);
    for (int w = w0; w < w1; ++w) {
      uint32_t bits = sel[w];
      uint32_t e = eqb[w];
      while (e && take > 0) {
        const uint32_t low = e & (0u - e);
        bits |= low;
        e ^= low;
        --take;
      }
      while (bits) {
        const int b = __ffs(bits) - 1;
        bits &= bits - 1;
        if (pos < topk) out[pos] = w * 32 + b;
        ++pos;
      }
    }
  }
  __syncthreads();   // S and the bitmaps are reused by the caller's next row
}

// What the finish kernel emits for a row once its k selected blocks are in out[0 .. k): the
// attention plan record of the one-token tile, or (the decode of one shard of a longer
// context, cand_score non-null) the (score, global block) candidates of the shard.
__device__ __forceinline__ void finish_emit(int32_t* rec, const PlanLayout& pl, int32_t* out,
                                            int k, int c, int p, const float* row_scores,
                                            float* cand_score_row, int32_t block0) {
  if (cand_score_row == nullptr) {
    write_decode_plan(rec, pl, out, k, c, p);
    return;
  }
  for (int j = threadIdx.x; j < k; j += blockDim.x) {
    const int i = out[j];
    cand_score_row[j] = row_scores[i];
    out[j] = i + block0;
  }
}

// Shared memory: TopkShared, then cap candidates (uint64), then two bitmaps of n_max bits.
// Besides idx/cnt, the finish kernel writes each row's attention plan record (one-token tile),
// or, for a shard (cand_score non-null), the selected blocks' scores and global block ids.
__global__ void __launch_bounds__(kTopkThreads) k_topk_finish(
    const float* __restrict__ scores, int64_t ld, const int32_t* __restrict__ n_c, int topk,
    int cap, int n_max, const uint32_t* __restrict__ hist, const int32_t* __restrict__ cand_cnt,
    const uint64_t* __restrict__ cand, const int32_t* __restrict__ rinfo,
    int32_t* __restrict__ idx, int32_t* __restrict__ cnt, const int32_t* __restrict__ len,
    PlanLayout pl, int32_t* __restrict__ plan, float* __restrict__ cand_score,
    int32_t block0) {
  pdl_trigger();
  pdl_wait();
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  TopkShared& S = *reinterpret_cast<TopkShared*>(smem_raw);
  uint64_t* c = reinterpret_cast<uint64_t*>(smem_raw + kTopkSharedBytes);
  const int nwords = (n_max + 31) / 32;
  uint32_t* sel = reinterpret_cast<uint32_t*>(c + cap);
  uint32_t* eqb = sel + nwords;
  const int tid = threadIdx.x;
  const int r = blockIdx.x;
  const int n = n_c[r];
  int32_t* out = idx + static_cast<int64_t>(r) * topk;
  int32_t* rec = plan != nullptr ? plan + static_cast<int64_t>(r) * pl.stride : nullptr;
  const int p = len[r] - 1;
  const float* row_scores = scores + static_cast<int64_t>(r) * ld;
  float* cs = cand_score != nullptr ? cand_score + static_cast<int64_t>(r) * topk : nullptr;
  if (n <= topk) {
    for (int i = tid; i < topk; i += blockDim.x) out[i] = i < n ? i : -1;
    if (tid == 0) cnt[r] = n < 0 ? 0 : n;
    __syncthreads();
    finish_emit(rec, pl, out, n < 0 ? 0 : n, n < 0 ? 0 : n, p, row_scores, cs, block0);
    return;
  }
  const uint32_t* h = hist + static_cast<int64_t>(r) * 4096;
  // the threshold bin and its counts, as the collect kernel found them in the histogram
  const uint32_t b1 = static_cast<uint32_t>(rinfo[4 * r]);
  const int above = rinfo[4 * r + 1];
  const int in_b1 = rinfo[4 * r + 2];
  const int C = cand_cnt[r];
  if (above + in_b1 > cap || C > cap) {
    // the candidates did not fit: full-row radix select on the scores in global memory
    topk_row(row_scores, n, topk, h, out, S);
    if (tid == 0) cnt[r] = topk;
    __syncthreads();
    finish_emit(rec, pl, out, topk, n, p, row_scores, cs, block0);
    return;
  }
  for (int i = tid; i < C; i += blockDim.x) c[i] = cand[static_cast<int64_t>(r) * cap + i];
  topk_select_candidates(S, c, C, b1, topk - above, sel, eqb, (n + 31) / 32, topk, out);
  if (tid == 0) cnt[r] = topk;
  __syncthreads();
  finish_emit(rec, pl, out, topk, n, p, row_scores, cs, block0);
}

// Step a3 on score rows, one CTA per row (grid-strided): pass 1 reads the row and builds the
// first-digit histogram (key bits 31..20); pass 2 reads it again (from L2) and collects the
// composites of the keys at or above the threshold bin b1 into shared memory; the exact select
// and the ordered output then run on those candidates (topk_select_candidates).  A row whose
// candidates would exceed `cap` takes the full-row select (topk_row).  Rows whose start is
// 16-byte aligned (ld a multiple of 4) are read as float4.
// Shared memory: TopkShared, then cap candidates (uint64), then two bitmaps of n_max bits.
__global__ void __launch_bounds__(kTopkThreads, 4) k_topk(const float* __restrict__ scores, int64_t ld,
                                                       const int32_t* __restrict__ n_c, int64_t rows,
                                                       int topk, int cap, int n_max,
                                                       int32_t* __restrict__ idx,
                                                       int32_t* __restrict__ cnt,
                                                       const int32_t* __restrict__ rinfo) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  TopkShared& S = *reinterpret_cast<TopkShared*>(smem_raw);
  uint64_t* c = reinterpret_cast<uint64_t*>(smem_raw + kTopkSharedBytes);
  uint32_t* sel = reinterpret_cast<uint32_t*>(c + cap);
  uint32_t* eqb = sel + (n_max + 31) / 32;
  __shared__ int s_cc;
  const int tid = threadIdx.x, lane = tid & 31;
  const bool vec = (ld & 3) == 0;
  for (int64_t r = blockIdx.x; r < rows; r += gridDim.x) {
    const int n = n_c[r];
    int32_t* out = idx + r * topk;
    if (n <= topk) {
      for (int i = tid; i < topk; i += blockDim.x) out[i] = i < n ? i : -1;
      if (tid == 0) cnt[r] = n < 0 ? 0 : n;
      continue;
    }
    const float* src = scores + r * ld;
    uint32_t b1;
    int above, in_b1;
    if (rinfo != nullptr) {
      // the indexer counted the row's first digit and found its threshold bin (select_mode 1)
      if (tid == 0) s_cc = 0;
      b1 = static_cast<uint32_t>(rinfo[4 * r]);
      above = rinfo[4 * r + 1];
      in_b1 = rinfo[4 * r + 2];
      __syncthreads();
    } else {
    // ---- pass 1: first-digit histogram ----
    clear_bins(S.hist, kTopkBins);
    if (tid == 0) s_cc = 0;
    __syncthreads();
    for (int base = 0; base < n; base += 4 * kTopkThreads) {
      const int i0 = base + 4 * tid;
      float x[4];
      if (vec && i0 + 3 < n) {
        const float4 f = *reinterpret_cast<const float4*>(src + i0);
        x[0] = f.x; x[1] = f.y; x[2] = f.z; x[3] = f.w;
      } else {
#pragma unroll
        for (int q = 0; q < 4; ++q) x[q] = i0 + q < n ? src[i0 + q] : 0.f;
      }
      // plain shared atomics: the hardware merges lanes that hit the same bin more cheaply
      // than grouping them first (__match_any_sync) for this row-at-a-time access pattern
#pragma unroll
      for (int q = 0; q < 4; ++q)
        if (i0 + q < n) atomicAdd(&S.hist[float_key(x[q]) >> 20], 1u);
    }
    __syncthreads();
    b1 = static_cast<uint32_t>(topk_find_bin(S, S.hist, kTopkBins, topk, &above, &in_b1));
    }
    if (above + in_b1 > cap) {
      topk_row(src, n, topk, nullptr, out, S);
      if (tid == 0) cnt[r] = topk;
      continue;
    }
    // ---- pass 2: candidates at or above bin b1 ----
    for (int base = 0; base < n; base += 4 * kTopkThreads) {
      const int i0 = base + 4 * tid;
      float x[4];
      if (vec && i0 + 3 < n) {
        const float4 f = *reinterpret_cast<const float4*>(src + i0);
        x[0] = f.x; x[1] = f.y; x[2] = f.z; x[3] = f.w;
      } else {
#pragma unroll
        for (int q = 0; q < 4; ++q) x[q] = i0 + q < n ? src[i0 + q] : 0.f;
      }
      uint32_t take = 0;
#pragma unroll
      for (int q = 0; q < 4; ++q)
        if (i0 + q < n && (float_key(x[q]) >> 20) >= b1) take |= 1u << q;
      int tot;
      const int ex = warp_count_scan(__popc(take), &tot);
      int slot = 0;
      if (tot) {
        if (lane == 0) slot = atomicAdd(&s_cc, tot);
        slot = __shfl_sync(0xffffffffu, slot, 0) + ex;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          if (take & (1u << q)) {
            c[slot] = (static_cast<uint64_t>(float_key(x[q])) << 32) | static_cast<uint32_t>(i0 + q);
            ++slot;
          }
        }
      }
    }
    __syncthreads();
    topk_select_candidates(S, c, s_cc, b1, topk - above, sel, eqb, (n + 31) / 32, topk, out);
    if (tid == 0) cnt[r] = topk;
  }
}

// ---------------------------------------------------------------------------------------
constexpr int kPlanThreads = 256;

// kDecode: tile = sequence b, single token at p = len[b]-1, selection rows idx[b].
__global__ void __launch_bounds__(kPlanThreads) k_attn_plan(
    const int32_t* __restrict__ idx, const int32_t* __restrict__ cnt, int topk,
    const SeqMeta* __restrict__ meta, int num_seqs, int num_tiles, PlanLayout pl, int max_words,
    int32_t* __restrict__ plan, DevStatus st) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  uint32_t* bitmap = reinterpret_cast<uint32_t*>(smem_raw);          // max_words
  int* wpref = reinterpret_cast<int*>(bitmap + max_words);            // max_words
  uint32_t* masks = reinterpret_cast<uint32_t*>(wpref + max_words);   // R * umax/32
  __shared__ int sh[33];
  __shared__ int64_t s_row0;
  __shared__ int s_pos0, s_ntok;
  const int tid = threadIdx.x;
  const int mwords = pl.umax / 32;
  for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
    if (tid == 0) {
      const int s = find_seq_of_tile<true>(meta, num_seqs, tile);
      const int lt = tile - meta[s].attn_tile0;
      const int p0 = lt * pl.R;
      s_pos0 = p0;
      s_row0 = meta[s].tok0 + p0;
      const int rem = meta[s].len - p0;
      s_ntok = rem < pl.R ? rem : pl.R;
    }
    __syncthreads();
    const int ntok = s_ntok, pos0 = s_pos0;
    const int64_t row0 = s_row0;
    int32_t* rec = plan + static_cast<int64_t>(tile) * pl.stride;
    if (ntok <= 0 || pos0 < 0) {
      if (tid == 0) {
        rec[0] = 0;
        rec[1] = 0;
      }
      __syncthreads();
      continue;
    }
    const int c_last = (pos0 + ntok - 1) / kBlock;
    const int nwords = c_last / 32 + 1;
    if (nwords > max_words) {
      if (tid == 0) {
        report_error(st, kErrDevice, 300);
        rec[0] = 0;
        rec[1] = 0;
      }
      __syncthreads();
      continue;
    }
    for (int i = tid; i < nwords; i += blockDim.x) bitmap[i] = 0;
    for (int i = tid; i < pl.R * mwords; i += blockDim.x) masks[i] = 0;
    __syncthreads();
    // mark selected blocks and own blocks
    for (int r = 0; r < ntok; ++r) {
      const int c_r = (pos0 + r) / kBlock;
      const int n = cnt[row0 + r];
      const int32_t* ir = idx + (row0 + r) * topk;
      for (int j = tid; j < n; j += blockDim.x) {
        const int b = ir[j];
        if (b < 0 || b >= c_r) {
          report_error(st, kErrDevice, 301);
          continue;
        }
        atomicOr(&bitmap[b >> 5], 1u << (b & 31));
      }
      if (tid == 0) atomicOr(&bitmap[c_r >> 5], 1u << (c_r & 31));
    }
    __syncthreads();
    // prefix popcounts over bitmap words
    int carry = 0;
    for (int base = 0; base < nwords; base += blockDim.x) {
      const int w = base + tid;
      const int pc = w < nwords ? __popc(bitmap[w]) : 0;
      int tot;
      const int ex = block_excl_scan(pc, sh, &tot);
      if (w < nwords) wpref[w] = carry + ex;
      carry += tot;
    }
    __syncthreads();
    const int U = carry;
    if (U > pl.umax) {   // cannot happen for valid selections
      if (tid == 0) {
        report_error(st, kErrDevice, 302);
        rec[0] = 0;
        rec[1] = 0;
      }
      __syncthreads();
      continue;
    }
    int32_t* uni = rec + pl.union_off();
    for (int w = tid; w < nwords; w += blockDim.x) {
      uint32_t bits = bitmap[w];
      int pos = wpref[w];
      while (bits) {
        const int bit = __ffs(bits) - 1;
        bits &= bits - 1;
        uni[pos++] = w * 32 + bit;
      }
    }
    // masks and tails
    for (int r = 0; r < ntok; ++r) {
      const int c_r = (pos0 + r) / kBlock;
      const int n = cnt[row0 + r];
      const int32_t* ir = idx + (row0 + r) * topk;
      for (int j = tid; j <= n; j += blockDim.x) {
        int b = (j < n) ? ir[j] : c_r;
        if (b < 0 || b > c_r) continue;
        const int w = b >> 5;
        const int pos = wpref[w] + __popc(bitmap[w] & ((1u << (b & 31)) - 1u));
        atomicOr(&masks[r * mwords + (pos >> 5)], 1u << (pos & 31));
        if (j == n) rec[pl.tail_off() + r] = pos;
      }
    }
    __syncthreads();
    const int nq = (U + 31) / 32;
    uint32_t* mout = reinterpret_cast<uint32_t*>(rec + pl.mask_off());
    for (int i = tid; i < ntok * mwords; i += blockDim.x) {
      const int r = i / mwords, q = i % mwords;
      if (q < nq) mout[r * mwords + q] = masks[r * mwords + q];
    }
    if (tid == 0) {
      rec[0] = U;
      rec[1] = ntok;
      rec[2] = pos0;
    }
    __syncthreads();
  }
}

// ---------------------------------------------------------------------------------------
// Decode: merge the split partials of each (sequence, head) by log-sum-exp.
//   partial O (unnormalised, fp32) [B][2][splits][12][128]; m (log2 domain), l [B][2][splits][12]
__global__ void k_decode_combine(const float* __restrict__ part_o, const float* __restrict__ part_m,
                                 const float* __restrict__ part_l, int batch, int splits,
                                 __nv_bfloat16* __restrict__ out) {
  pdl_trigger();
  pdl_wait();
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= batch * kHeads) return;
  const int b = warp / kHeads, h = warp % kHeads, g = h / kGroup, hr = h % kGroup;
  const int64_t base = (static_cast<int64_t>(b) * 2 + g) * splits;
  float M = -INFINITY;
  for (int s = 0; s < splits; ++s) M = fmaxf(M, part_m[(base + s) * kGroup + hr]);
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  float L = 0.f;
  for (int s = 0; s < splits; ++s) {
    const float m = part_m[(base + s) * kGroup + hr];
    const float f = (m == -INFINITY) ? 0.f : exp2f(m - M);
    L += f * part_l[(base + s) * kGroup + hr];
    const float4 o = reinterpret_cast<const float4*>(
        part_o + ((base + s) * kGroup + hr) * kHeadDim)[lane];
    acc[0] += f * o.x;
    acc[1] += f * o.y;
    acc[2] += f * o.z;
    acc[3] += f * o.w;
  }
  const float inv = L > 0.f ? 1.f / L : 0.f;
  uint2 pk;
  pk.x = pack_bf16x2(acc[0] * inv, acc[1] * inv);
  pk.y = pack_bf16x2(acc[2] * inv, acc[3] * inv);
  reinterpret_cast<uint2*>(out + (static_cast<int64_t>(b) * kHeads + h) * kHeadDim)[lane] = pk;
}

// ---------------------------------------------------------------------------------------
// Context-sharded decode.  A sequence's context is split over shards (caches of consecutive
// tokens, each starting on a 512-token boundary, one per GPU); every shard proposes the top-k
// of its own candidate blocks, and the selection is the top-k of their union.

// Merge: the shards' (score, global block) candidates of one sequence -> the sequence's
// selection, larger score first and the lower block among equal scores, emitted in ascending
// block order (the same order as a selection over the whole context).  One CTA per sequence.
// cs/ci [shards][batch][topk], cc [shards][batch].  Shared memory: TopkShared, then
// shards * topk composites, then two bitmaps of nwords words (global blocks < 32 nwords).
constexpr int kMaxShards = 64;
__global__ void __launch_bounds__(kTopkThreads) k_merge_candidates(
    const float* __restrict__ cs, const int32_t* __restrict__ ci, const int32_t* __restrict__ cc,
    int shards, int batch, int topk, int nwords, int32_t* __restrict__ idx,
    int32_t* __restrict__ cnt, DevStatus st) {
  pdl_trigger();
  pdl_wait();
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  TopkShared& S = *reinterpret_cast<TopkShared*>(smem_raw);
  uint64_t* c = reinterpret_cast<uint64_t*>(smem_raw + kTopkSharedBytes);
  uint32_t* sel = reinterpret_cast<uint32_t*>(c + static_cast<int64_t>(shards) * topk);
  uint32_t* eqb = sel + nwords;
  __shared__ int s_off[kMaxShards + 1];
  const int b = blockIdx.x, tid = threadIdx.x;
  if (tid == 0) {
    int o = 0;
    for (int r = 0; r < shards; ++r) {
      s_off[r] = o;
      int k = cc[static_cast<int64_t>(r) * batch + b];
      if (k < 0 || k > topk) {
        report_error(st, kErrDevice, 310);
        k = k < 0 ? 0 : topk;
      }
      o += k;
    }
    s_off[shards] = o;
  }
  __syncthreads();
  const int C = s_off[shards];
  for (int r = 0; r < shards; ++r) {
    const int k = s_off[r + 1] - s_off[r];
    for (int j = tid; j < k; j += blockDim.x) {
      const int64_t e = (static_cast<int64_t>(r) * batch + b) * topk + j;
      int blk = ci[e];
      uint32_t key = float_key(cs[e]);
      if (blk < 0 || blk >= 32 * nwords) {   // never followed: reported, ranked last
        report_error(st, kErrDevice, 311);
        blk = 0;
        key = 0u;
      }
      c[s_off[r] + j] = (static_cast<uint64_t>(key) << 32) | static_cast<uint32_t>(blk);
    }
  }
  const int K = C < topk ? C : topk;
  int32_t* out = idx + static_cast<int64_t>(b) * topk;
  for (int j = K + tid; j < topk; j += blockDim.x) out[j] = -1;
  if (tid == 0) cnt[b] = K;
  if (K == 0) return;   // uniform
  clear_bins(S.hist, kTopkBins);
  __syncthreads();
  for (int i = tid; i < C; i += blockDim.x)
    atomicAdd(&S.hist[static_cast<uint32_t>(c[i] >> 32) >> 20], 1u);
  __syncthreads();
  int above;
  const uint32_t b1 = static_cast<uint32_t>(topk_find_bin(S, S.hist, kTopkBins, K, &above));
  topk_select_candidates(S, c, C, b1, K - above, sel, eqb, nwords, K, out);
}

// Attention plan of one shard (one-token tile per sequence): the selected blocks (ascending
// global ids) that lie in the shard's blocks [block0, block0 + nblk), as local ids, followed by
// the query's own block when the shard holds it; every union block is attended.  One CTA per
// sequence.
__global__ void __launch_bounds__(kPlanThreads) k_shard_plan(
    const int32_t* __restrict__ sel_idx, const int32_t* __restrict__ sel_cnt, int topk,
    const int32_t* __restrict__ glen, int32_t block0, int32_t nblk, PlanLayout pl,
    int32_t* __restrict__ plan, DevStatus st) {
  pdl_trigger();
  pdl_wait();
  __shared__ int s_lo, s_hi;
  const int b = blockIdx.x, tid = threadIdx.x;
  const int p = glen[b] - 1;
  const int own = p >= 0 ? p / kBlock : -1;
  int n = sel_cnt[b];
  if (n < 0 || n > topk) {
    if (tid == 0) report_error(st, kErrDevice, 312);
    n = n < 0 ? 0 : topk;
  }
  const int32_t* s = sel_idx + static_cast<int64_t>(b) * topk;
  if (tid == 0) {
    int lo = 0, hi = n;   // first entry >= block0
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (s[mid] < block0) lo = mid + 1; else hi = mid;
    }
    int lo2 = lo, hi2 = n;   // first entry >= block0 + nblk
    while (lo2 < hi2) {
      const int mid = (lo2 + hi2) >> 1;
      if (s[mid] < block0 + nblk) lo2 = mid + 1; else hi2 = mid;
    }
    s_lo = lo;
    s_hi = lo2;
  }
  __syncthreads();
  const int lo = s_lo, k = s_hi - s_lo;
  const bool own_here = own >= block0 && own < block0 + nblk;
  const int U = k + (own_here ? 1 : 0);
  int32_t* rec = plan + static_cast<int64_t>(b) * pl.stride;
  int32_t* uni = rec + pl.union_off();
  for (int j = tid; j < k; j += blockDim.x) {
    const int blk = s[lo + j];
    if (blk >= own) report_error(st, kErrDevice, 313);   // not a candidate of the query
    uni[j] = blk - block0;
  }
  uint32_t* m = reinterpret_cast<uint32_t*>(rec + pl.mask_off());
  for (int q = tid; q < (U + 31) / 32; q += blockDim.x) {
    const int rem = U - 32 * q;
    m[q] = rem >= 32 ? 0xffffffffu : ((1u << rem) - 1u);
  }
  if (tid == 0) {
    if (own_here) uni[k] = own - block0;
    rec[0] = U;
    rec[1] = 1;
    rec[2] = p;
    rec[pl.tail_off()] = own_here ? k : -1000000;   // no own block here: nothing to hide
  }
}

// Combine: the shards' partial softmaxes of every (sequence, head), by log-sum-exp.
//   part_o [shards][B][24][128] (unnormalised, fp32), part_m (log2 domain), part_l
//   [shards][B][24].  One warp per (sequence, head), 4 dims per lane.
__global__ void k_combine_shards(const float* __restrict__ part_o, const float* __restrict__ part_m,
                                 const float* __restrict__ part_l, int batch, int shards,
                                 __nv_bfloat16* __restrict__ out) {
  pdl_trigger();
  pdl_wait();
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= batch * kHeads) return;
  const int64_t per_shard = static_cast<int64_t>(batch) * kHeads;
  float M = -INFINITY;
  for (int r = 0; r < shards; ++r) M = fmaxf(M, part_m[r * per_shard + warp]);
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  float L = 0.f;
  for (int r = 0; r < shards; ++r) {
    const float m = part_m[r * per_shard + warp];
    const float f = (m == -INFINITY) ? 0.f : exp2f(m - M);
    L += f * part_l[r * per_shard + warp];
    const float4 o = reinterpret_cast<const float4*>(part_o + (r * per_shard + warp) * kHeadDim)[lane];
    acc[0] += f * o.x;
    acc[1] += f * o.y;
    acc[2] += f * o.z;
    acc[3] += f * o.w;
  }
  const float inv = L > 0.f ? 1.f / L : 0.f;
  uint2 pk;
  pk.x = pack_bf16x2(acc[0] * inv, acc[1] * inv);
  pk.y = pack_bf16x2(acc[2] * inv, acc[3] * inv);
  reinterpret_cast<uint2*>(out + static_cast<int64_t>(warp) * kHeadDim)[lane] = pk;
}

}  // namespace qsa
