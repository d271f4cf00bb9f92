// qsa_attn.cuh -- steps a4/a6: attention over the selected blocks plus the own block.
//
// One CTA handles one attention tile (up to R consecutive query tokens of a sequence, R = 1
// in decode) for one KV head g.  Its 128 tensor-core rows are (token, query head of group g)
// pairs: row = 12 * token + head, rows >= 12R are padding.  Keys are the tile's union of
// selected blocks and own blocks (see k_attn_plan), processed 32 blocks = 128 keys per chunk.
//
// Per chunk i (S and P double-buffered in TMEM, K/V double-buffered in shared memory):
//   S = Q K^T        tcgen05, A = Q (smem, K-major), B = K chunk (smem, K-major), D in TMEM
//   softmax          one thread per row: mask keys the row's token did not select (and the
//                    own block's future tokens), online max in the log2 domain with lazy
//                    rescaling of O (only when the max grows by more than 2^8), P = exp2(.)
//                    written back over S in TMEM as bf16
//   O += P V         tcgen05, A = P (TMEM), B = V chunk (smem, MN-major), D = O in TMEM
// K/V rows are gathered per 4-token block with TMA boxes of 4 rows x 64 dims (no multicast).
//
// Warp roles: warps 0-3 softmax (warp w owns TMEM lanes 32w..32w+31), warp 4 TMA producer,
// warp 5 TMEM allocation + MMA issue.
#pragma once

#include "qsa_common.cuh"
#include "qsa_misc.cuh"

namespace qsa {

struct AttnCfg {
  static constexpr int kThreads = 192;
  static constexpr int kChunkBlocks = 32;
  static constexpr int kChunkKeys = 128;
  static constexpr int kQBytes = 128 * kHeadDim * 2;     // 32 KB (2 panels of 16 KB)
  static constexpr int kKVBytes = kChunkKeys * kHeadDim * 2;   // 32 KB per K or V tile
  static constexpr int kStages = 2;
  static constexpr int kQOff = 0;
  static constexpr int kKOff = kQBytes;                        // stage s: K at kKOff + s*64KB
  static constexpr int kStageBytes = 2 * kKVBytes;
  static constexpr int kBarOff = kKOff + kStages * kStageBytes;
  static constexpr int kNumBars = 1 + 2 * kStages + 2 + 2 + 1 + 1;
  static constexpr int kSmemBytes = kBarOff + kNumBars * 8 + 16 + 1024;
  static constexpr int kTmemCols = 512;                  // S0 [0,128) S1 [128,256) O [256,384)
  static constexpr uint32_t kIdescQK = idesc_bf16_f32(128, 128, 0, 0);
  static constexpr uint32_t kIdescPV = idesc_bf16_f32(128, 128, 0, 1);   // B = V is MN-major
};

struct AttnArgs {
  const int32_t* plan;     // tile records (PlanLayout)
  PlanLayout pl;
  const SeqMeta* meta;     // prefill
  int32_t num_seqs;
  int32_t decode;          // 1: decode (tile = sequence, KV from the block cache)
  int32_t splits;          // chunk splits per tile (decode), 1 for prefill
  int64_t cap_blocks;      // decode: capacity / 4
  __nv_bfloat16* out;      // prefill: [T][24][128]
  float* part_o;           // decode: [B][2][splits][12][128]
  float* part_m;           // decode: [B][2][splits][12]
  float* part_l;
  DevStatus st;
};

__device__ __forceinline__ uint32_t spread_nibbles(uint32_t byte) {
  // bit i of byte -> nibble i of the result set to 0xF
  uint32_t x = byte & 0xffu;
  x = (x | (x << 12)) & 0x000F000Fu;
  x = (x | (x << 6)) & 0x03030303u;
  x = (x | (x << 3)) & 0x11111111u;
  return x * 0xFu;
}

__global__ void __launch_bounds__(AttnCfg::kThreads, 1)
    k_sparse_attn(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_k,
                  const __grid_constant__ CUtensorMap tmap_v, AttnArgs args) {
  using C = AttnCfg;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  unsigned char* sQ = smem + C::kQOff;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
  uint64_t* q_full = bars;
  uint64_t* kv_full = bars + 1;
  uint64_t* kv_empty = kv_full + C::kStages;
  uint64_t* s_full = kv_empty + C::kStages;
  uint64_t* p_full = s_full + 2;
  uint64_t* pv_done = p_full + 2;
  uint64_t* mma_done = pv_done + 1;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(bars + C::kNumBars);
  volatile int* s_abort = reinterpret_cast<volatile int*>(s_tmem + 1);

  const int g = blockIdx.y;
  const int split = blockIdx.z;
  const int tile = blockIdx.x;
  const int32_t* rec = args.plan + static_cast<int64_t>(tile) * args.pl.stride;
  const int U = rec[0];
  const int ntok = rec[1];
  const int R = args.pl.R;
  const int nchunks_all = (U + C::kChunkBlocks - 1) / C::kChunkBlocks;
  int c_begin = 0, c_end = nchunks_all;
  if (args.decode) {
    const int per = (nchunks_all + args.splits - 1) / args.splits;
    c_begin = split * per;
    c_end = c_begin + per < nchunks_all ? c_begin + per : nchunks_all;
  }
  const int nchunks = c_end > c_begin ? c_end - c_begin : 0;

  // where this tile's tokens live
  int64_t tok_row0 = 0;   // global token row (prefill) / sequence (decode) of token 0
  int pos0 = 0;           // position within the sequence of token 0
  int64_t kv_row_base = 0;
  if (args.decode) {
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

  if (nchunks == 0 || ntok == 0) {
    // decode split without keys: write an empty partial
    if (args.decode && ntok > 0 && threadIdx.x < kGroup) {
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
    for (int i = 0; i < C::kStages; ++i) {
      mbar_init(&kv_full[i], 1);
      mbar_init(&kv_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], 4);
    }
    mbar_init(pv_done, 1);
    mbar_init(mma_done, 1);
    *s_abort = 0;
    fence_mbar_init();
  }
  // zero the rows of Q below the TMA box (rows 12R..127 are never written by TMA)
  {
    const int box_rows = kGroup * R;
    const int pad_rows = 128 - box_rows;
    for (int i = threadIdx.x; i < pad_rows * 16; i += blockDim.x) {
      const int r = box_rows + i / 16, c = i % 16;   // 16 x 16 B per row (both panels)
      const int panel = c / 8, cc = c % 8;
      *reinterpret_cast<uint4*>(sQ + panel * 16384 + r * 128 + cc * 16) = make_uint4(0, 0, 0, 0);
    }
    fence_proxy_async_smem();
  }
  if (warp == 5) {
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

  if (warp == 4) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      prefetch_tmap(&tmap_q);
      prefetch_tmap(&tmap_k);
      prefetch_tmap(&tmap_v);
      const uint32_t qbytes = 2u * kGroup * R * 128u;   // full box, out-of-range rows zero-filled
      mbar_arrive_expect_tx(q_full, qbytes);
      // Q box: 64 dims x 12 heads x ntok tokens, rows land as 12*token + head
      for (int half = 0; half < 2; ++half)
        tma_load_3d(sQ + half * 16384, &tmap_q, half * 64, g * kGroup,
                    static_cast<int32_t>(tok_row0), q_full);
    }
    __syncwarp();
    int issued = 0;
    for (int i = 0; i < nchunks; ++i) {
      const int s = i % C::kStages;
      bool ok = true;
      if (lane == 0) ok = mbar_wait(&kv_empty[s], ((i / C::kStages) & 1) ^ 1, s_abort, args.st, 20);
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      if (!ok) break;
      if (lane == 0) mbar_arrive_expect_tx(&kv_full[s], 2u * C::kKVBytes);
      __syncwarp();
      const int upos = (c_begin + i) * C::kChunkBlocks + lane;
      const int blk = upos < U ? uni[upos] : uni[0];   // padding slots repeat a real block
      unsigned char* sK = smem + C::kKOff + s * C::kStageBytes;
      unsigned char* sV = sK + C::kKVBytes;
      if (args.decode) {
        const int32_t row = static_cast<int32_t>(kv_row_base + static_cast<int64_t>(blk) * kBlock);
        for (int half = 0; half < 2; ++half) {
          tma_load_2d(sK + half * 16384 + lane * 512, &tmap_k, half * 64, row, &kv_full[s]);
          tma_load_2d(sV + half * 16384 + lane * 512, &tmap_v, half * 64, row, &kv_full[s]);
        }
      } else {
        const int32_t row = static_cast<int32_t>(kv_row_base + static_cast<int64_t>(blk) * kBlock);
        for (int half = 0; half < 2; ++half) {
          tma_load_2d(sK + half * 16384 + lane * 512, &tmap_k, g * kHeadDim + half * 64, row,
                      &kv_full[s]);
          tma_load_2d(sV + half * 16384 + lane * 512, &tmap_v, g * kHeadDim + half * 64, row,
                      &kv_full[s]);
        }
      }
      ++issued;
    }
    if (lane == 0 && *s_abort) {
      const int from = issued > C::kStages ? issued - C::kStages : 0;
      for (int j = from; j < issued; ++j) mbar_drain(&kv_full[j % C::kStages], (j / C::kStages) & 1);
      mbar_drain(q_full, 0);
    }
  } else if (warp == 5) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      const uint32_t sQ0 = smem_u32(sQ);
      bool ok = mbar_wait(q_full, 0, s_abort, args.st, 21);
      auto issue_pv = [&](int j) -> bool {
        const int bj = j & 1;
        if (!mbar_wait(&p_full[bj], (j >> 1) & 1, s_abort, args.st, 22)) return false;
        tc_fence_after();
        const uint32_t sV0 = smem_u32(smem + C::kKOff + (j % C::kStages) * C::kStageBytes + C::kKVBytes);
#pragma unroll
        for (int k = 0; k < C::kChunkKeys / 16; ++k) {
          // B = V chunk, MN-major: 16 keys per step = 2048 bytes; next 64 dims at +16 KB
          const uint64_t db = smem_desc_sw128(sV0 + 2048 * k, 16384, 1024);
          umma_ts(tmem_O, tmem + bj * 128 + 8 * k, db, C::kIdescPV, (j > 0 || k > 0) ? 1u : 0u);
        }
        umma_commit(&kv_empty[j % C::kStages]);
        umma_commit(pv_done);
        return true;
      };
      for (int i = 0; ok && i < nchunks; ++i) {
        const int b = i & 1;
        const int s = i % C::kStages;
        if (!mbar_wait(&kv_full[s], (i / C::kStages) & 1, s_abort, args.st, 23)) break;
        tc_fence_after();
        const uint32_t sK0 = smem_u32(smem + C::kKOff + s * C::kStageBytes);
#pragma unroll
        for (int k = 0; k < kHeadDim / 16; ++k) {
          const int half = k >> 2, kk = k & 3;
          const uint64_t da = smem_desc_sw128(sQ0 + half * 16384 + 32 * kk, 0, 1024);
          const uint64_t db = smem_desc_sw128(sK0 + half * 16384 + 32 * kk, 0, 1024);
          umma_ss(tmem + b * 128, da, db, C::kIdescQK, k > 0 ? 1u : 0u);
        }
        umma_commit(&s_full[b]);
        if (i > 0 && !issue_pv(i - 1)) break;
        if (i == nchunks - 1) issue_pv(i);
      }
      umma_commit(mma_done);
      mbar_drain(mma_done, 0);
    }
  } else {
    // ---------------- softmax (warps 0-3) ----------------
    const int row = warp * 32 + lane;
    const int valid_rows = kGroup * ntok;
    const bool row_ok = row < valid_rows;
    const bool warp_active = warp * 32 < valid_rows;
    const int tr = row_ok ? row / kGroup : 0;
    const int hr = row % kGroup;
    const int pos = pos0 + tr;
    const int tail_u = row_ok ? rec[args.pl.tail_off() + tr] : -1;
    const int tail_last = pos % kBlock;   // keys 0..tail_last of the own block are visible
    const float sl2 = 1.4426950408889634f * 0.08838834764831845f;   // log2(e)/sqrt(128)
    float m = -INFINITY, l = 0.f;
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    bool ok = true;
    for (int i = 0; i < nchunks; ++i) {
      const int b = i & 1;
      const bool got = mbar_wait(&s_full[b], (i >> 1) & 1, s_abort, args.st, 24);
      if (__any_sync(0xffffffffu, !got)) {   // also reconverges the warp
        ok = false;
        break;
      }
      tc_fence_after();
      if (warp_active) {
        const int q = c_begin + i;
        uint32_t mword = row_ok ? masks[tr * mwords + q] : 0u;
        uint32_t km[4];
#pragma unroll
        for (int w4 = 0; w4 < 4; ++w4) km[w4] = spread_nibbles(mword >> (8 * w4));
        const int tu = tail_u - q * C::kChunkBlocks;
        if (tu >= 0 && tu < C::kChunkBlocks) {
          // hide the own block's keys after the query position
          const int key0 = tu * 4;
          for (int kk = tail_last + 1; kk < 4; ++kk) {
            const int key = key0 + kk;
            km[key >> 5] &= ~(1u << (key & 31));
          }
        }
        uint32_t sv[128];
        const uint32_t ts = tmem + lane_base + b * 128;
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld32(ts + 32 * c, sv + 32 * c);
        tmem_wait_ld();
        float mx = -INFINITY;
#pragma unroll
        for (int j = 0; j < 128; ++j) {
          const bool v = (km[j >> 5] >> (j & 31)) & 1u;
          const float x = v ? __uint_as_float(sv[j]) * sl2 : -INFINITY;
          sv[j] = __float_as_uint(x);
          mx = fmaxf(mx, x);
        }
        const float m_cand = fmaxf(m, mx);
        const bool need = m_cand > m + 8.f || (m == -INFINITY && m_cand > -INFINITY);
        if (__any_sync(0xffffffffu, need)) {
          const float alpha = (m == -INFINITY) ? 0.f : exp2f(m - m_cand);
          if (i > 0) {
            // O holds PV of chunks < i-1 and maybe i-1: wait until chunk i-1 is in, rescale
            if (!mbar_wait(pv_done, (i - 1) & 1, s_abort, args.st, 25)) {
              ok = false;
            }
            if (__any_sync(0xffffffffu, !ok)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t to = tmem_O + lane_base;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              uint32_t ov[32];
              tmem_ld32(to + 32 * c, ov);
              tmem_wait_ld();
#pragma unroll
              for (int j = 0; j < 32; ++j) ov[j] = __float_as_uint(__uint_as_float(ov[j]) * alpha);
              tmem_st32(to + 32 * c, ov);
            }
          }
          l *= alpha;
          m = m_cand;
        }
        const float mref = (m == -INFINITY) ? 0.f : m;
        float lsum = 0.f;
        uint32_t pk[64];
#pragma unroll
        for (int j = 0; j < 64; ++j) {
          const float p0 = exp2f(__uint_as_float(sv[2 * j]) - mref);
          const float p1 = exp2f(__uint_as_float(sv[2 * j + 1]) - mref);
          lsum += p0 + p1;
          pk[j] = pack_bf16x2(p0, p1);
        }
        l += lsum;
        tmem_st32(ts, pk);
        tmem_st32(ts + 32, pk + 32);
        tmem_wait_st();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[b]);
    }
    if (ok && nchunks > 0) {
      const bool got = mbar_wait(pv_done, (nchunks - 1) & 1, s_abort, args.st, 26);
      if (!__any_sync(0xffffffffu, !got)) {
        tc_fence_after();
        if (warp_active) {
          const uint32_t to = tmem_O + lane_base;
          uint32_t ov[128];
#pragma unroll
          for (int c = 0; c < 4; ++c) tmem_ld32(to + 32 * c, ov + 32 * c);
          tmem_wait_ld();
          if (row_ok) {
            if (!args.decode) {
              const float inv = l > 0.f ? 1.f / l : 0.f;
              __nv_bfloat16* o = args.out + ((tok_row0 + tr) * kHeads + g * kGroup + hr) * kHeadDim;
#pragma unroll
              for (int c = 0; c < 16; ++c) {
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
              args.part_m[pr] = m;
              args.part_l[pr] = l;
              float4* po = reinterpret_cast<float4*>(args.part_o + pr * kHeadDim);
#pragma unroll
              for (int c = 0; c < 32; ++c)
                po[c] = make_float4(__uint_as_float(ov[4 * c]), __uint_as_float(ov[4 * c + 1]),
                                    __uint_as_float(ov[4 * c + 2]), __uint_as_float(ov[4 * c + 3]));
            }
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

}  // namespace qsa
