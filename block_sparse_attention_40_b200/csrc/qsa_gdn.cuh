// qsa_gdn.cuh -- the Gated DeltaNet linear-attention layer (the three of every four
// token-mixing layers around QSA), chunked.
//
// Per sequence and head, the state S (d_v x d_k, fp32) starts at zero, and each token t
// with gate alpha_t = exp(log_alpha_t) and writing strength beta_t updates it as
//     S_t = alpha_t S_{t-1} + beta_t (v_t - alpha_t S_{t-1} k_t) k_t^T,    o_t = S_t q_t
// (the gated delta rule; the pages name the layer, a gated linear recurrence over a compact
// state, but their table of its parameters did not survive extraction).
//
// Chunked form, for a chunk of C tokens entered with state S0, g_t the running sum of the
// chunk's log gates (g_0 = log_alpha_0) and u_t = beta_t (v_t - alpha_t S_{t-1} k_t) the
// value each token writes:
//     U   = (I + diag(beta) A)^-1 diag(beta) (V - diag(e^g) K S0^T),
//           A_tj = e^(g_t - g_j) k_t.k_j  for j < t      (forward substitution, row by row)
//     O   = diag(e^g) Q S0^T + M U,   M_tj = e^(g_t - g_j) q_t.k_j  for j <= t
//     S_C = e^(g_C) S0 + U^T diag(e^(g_C - g)) K
// One CTA of 512 threads per (sequence, head) walks the sequence's chunks of 64 tokens in
// order; the state (held transposed, k-major) and the chunk's tiles stay in shared memory,
// all in fp32 on the FMA pipes.  log_alpha is clamped at -87 (alpha below about 1.6e-38 acts
// as a full reset), which keeps the differences g_t - g_j finite.

#pragma once

#include "qsa_common.cuh"

namespace qsa {

constexpr int kGdnDim = 128;      // d_k = d_v
constexpr int kGdnChunk = 64;
constexpr int kGdnThreads = 512;
constexpr int kGdnKStride = kGdnDim + 4;   // K rows padded: 16-byte rows, 4-way at most on column stores
constexpr float kGdnMinLogAlpha = -87.f;

// Operands are laid out so that every product reads them as float4: K and Q also held
// transposed (k-major, tokens contiguous), so a thread's four rows arrive in one broadcast.
struct GdnSmem {
  float st[kGdnDim * kGdnDim];          // S^T: st[k][v]
  float k[kGdnChunk * kGdnKStride];     // K rows (padded): k[t][d]
  float kt[kGdnDim * kGdnChunk];        // K^T: kt[d][t]
  float qt[kGdnDim * kGdnChunk];        // Q^T: qt[d][t]
  float v[kGdnChunk * kGdnDim];         // V, then V - diag(e^g) K S0^T, then U
  float a[kGdnChunk * kGdnChunk];       // A (strictly lower)
  float m[kGdnChunk * kGdnChunk];       // M (lower, diagonal included)
  float g[kGdnChunk];                   // running log gate
  float beta[kGdnChunk];
  float wk[kGdnChunk];                  // e^(g_C - g_t)
};
constexpr int kGdnSmemBytes = static_cast<int>(sizeof(GdnSmem));
static_assert(kGdnSmemBytes <= 227 * 1024, "shared memory per CTA");

struct GdnArgs {
  const __nv_bfloat16* q;   // [T][H][128]
  const __nv_bfloat16* k;
  const __nv_bfloat16* v;
  const float* log_alpha;   // [T][H]
  const float* beta;        // [T][H]
  const int32_t* cu;        // [S+1]
  int32_t heads;
  __nv_bfloat16* out;       // [T][H][128]
  float* final_state;       // [S][H][128 (v)][128 (k)] or null
};

__device__ __forceinline__ float bf16_bits_to_float(uint32_t b) { return __uint_as_float(b << 16); }

// Rows t < n of the chunk starting at token t0 into shared memory (fp32); rows n..63 are
// zero with beta 0 and log gate 0, so they neither write nor decay the state.
__device__ __forceinline__ void gdn_load_chunk(const GdnArgs& a, GdnSmem& S, int h, int64_t t0,
                                               int n) {
  const int tid = threadIdx.x;
  // q and k: lanes take consecutive tokens (so the transposed stores are conflict-free);
  // v: lanes take consecutive 8-value groups of a row.  1024 groups of 8 bf16 per matrix.
  for (int e = tid; e < kGdnChunk * (kGdnDim / 8); e += kGdnThreads) {
    const int t = e % kGdnChunk, d0 = (e / kGdnChunk) * 8;
    uint4 rq = make_uint4(0u, 0u, 0u, 0u), rk = rq;
    if (t < n) {
      const int64_t off = ((t0 + t) * a.heads + h) * kGdnDim + d0;
      rq = *reinterpret_cast<const uint4*>(a.q + off);
      rk = *reinterpret_cast<const uint4*>(a.k + off);
    }
    const uint32_t wq[4] = {rq.x, rq.y, rq.z, rq.w}, wk[4] = {rk.x, rk.y, rk.z, rk.w};
    float kf[8];
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      S.qt[(d0 + 2 * p) * kGdnChunk + t] = bf16_bits_to_float(wq[p] & 0xffffu);
      S.qt[(d0 + 2 * p + 1) * kGdnChunk + t] = bf16_bits_to_float(wq[p] >> 16);
      kf[2 * p] = bf16_bits_to_float(wk[p] & 0xffffu);
      kf[2 * p + 1] = bf16_bits_to_float(wk[p] >> 16);
    }
#pragma unroll
    for (int p = 0; p < 8; ++p) S.kt[(d0 + p) * kGdnChunk + t] = kf[p];
    float4* kr = reinterpret_cast<float4*>(&S.k[t * kGdnKStride + d0]);
    kr[0] = make_float4(kf[0], kf[1], kf[2], kf[3]);
    kr[1] = make_float4(kf[4], kf[5], kf[6], kf[7]);
  }
  for (int e = tid; e < kGdnChunk * (kGdnDim / 8); e += kGdnThreads) {
    const int t = e / (kGdnDim / 8), d0 = (e % (kGdnDim / 8)) * 8;
    uint4 rv = make_uint4(0u, 0u, 0u, 0u);
    if (t < n) rv = *reinterpret_cast<const uint4*>(a.v + ((t0 + t) * a.heads + h) * kGdnDim + d0);
    const uint32_t wv[4] = {rv.x, rv.y, rv.z, rv.w};
    float4* vr = reinterpret_cast<float4*>(&S.v[t * kGdnDim + d0]);
    vr[0] = make_float4(bf16_bits_to_float(wv[0] & 0xffffu), bf16_bits_to_float(wv[0] >> 16),
                        bf16_bits_to_float(wv[1] & 0xffffu), bf16_bits_to_float(wv[1] >> 16));
    vr[1] = make_float4(bf16_bits_to_float(wv[2] & 0xffffu), bf16_bits_to_float(wv[2] >> 16),
                        bf16_bits_to_float(wv[3] & 0xffffu), bf16_bits_to_float(wv[3] >> 16));
  }
  // gates: warp 0, two tokens a lane, an inclusive scan of the clamped log gates
  if (tid < 32) {
    float la[2], bt[2];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const int t = 2 * tid + r;
      la[r] = 0.f;
      bt[r] = 0.f;
      if (t < n) {
        const int64_t i = (t0 + t) * a.heads + h;
        la[r] = fmaxf(a.log_alpha[i], kGdnMinLogAlpha);
        bt[r] = a.beta[i];
      }
    }
    const float pair = la[0] + la[1];
    float incl = pair;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const float y = __shfl_up_sync(0xffffffffu, incl, o);
      if (tid >= o) incl += y;
    }
    const float before = incl - pair;
    S.g[2 * tid] = before + la[0];
    S.g[2 * tid + 1] = incl;
    S.beta[2 * tid] = bt[0];
    S.beta[2 * tid + 1] = bt[1];
  }
}

// grid (heads, sequences), kGdnThreads threads, kGdnSmemBytes of dynamic shared memory.
__global__ void __launch_bounds__(kGdnThreads, 1) k_gated_deltanet(GdnArgs a) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  GdnSmem& S = *reinterpret_cast<GdnSmem*>(smem_raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int h = blockIdx.x, s = blockIdx.y;
  const int64_t t_begin = a.cu[s], t_end = a.cu[s + 1];
  for (int e = tid; e < kGdnDim * kGdnDim; e += kGdnThreads) S.st[e] = 0.f;
  __syncthreads();
  for (int64_t t0 = t_begin; t0 < t_end; t0 += kGdnChunk) {
    const int n = static_cast<int>(t_end - t0 < kGdnChunk ? t_end - t0 : kGdnChunk);
    gdn_load_chunk(a, S, h, t0, n);
    __syncthreads();
    // ---- K S0^T and Q S0^T: rows 4 warp .. +3, value columns 4 lane .. +3 ----
    float qs[4][4];
    {
      float ak[4][4], aq[4][4];
#pragma unroll
      for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int c = 0; c < 4; ++c) ak[r][c] = aq[r][c] = 0.f;
#pragma unroll 4
      for (int kk = 0; kk < kGdnDim; ++kk) {
        const float4 s4 = *reinterpret_cast<const float4*>(&S.st[kk * kGdnDim + 4 * lane]);
        const float4 k4 = *reinterpret_cast<const float4*>(&S.kt[kk * kGdnChunk + 4 * warp]);
        const float4 q4 = *reinterpret_cast<const float4*>(&S.qt[kk * kGdnChunk + 4 * warp]);
        const float sv[4] = {s4.x, s4.y, s4.z, s4.w};
        const float kr[4] = {k4.x, k4.y, k4.z, k4.w}, qr[4] = {q4.x, q4.y, q4.z, q4.w};
#pragma unroll
        for (int r = 0; r < 4; ++r) {
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            ak[r][c] = fmaf(kr[r], sv[c], ak[r][c]);
            aq[r][c] = fmaf(qr[r], sv[c], aq[r][c]);
          }
        }
      }
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const int t = 4 * warp + r;
        const float gam = __expf(S.g[t]);
        float4* vp = reinterpret_cast<float4*>(&S.v[t * kGdnDim + 4 * lane]);
        float4 vv = *vp;
        vv.x -= gam * ak[r][0];
        vv.y -= gam * ak[r][1];
        vv.z -= gam * ak[r][2];
        vv.w -= gam * ak[r][3];
        *vp = vv;
#pragma unroll
        for (int c = 0; c < 4; ++c) qs[r][c] = gam * aq[r][c];
      }
    }
    // ---- A (strictly lower) and M (lower): rows 4 warp .. +3, columns 2 lane, 2 lane + 1 ----
    {
      float ka[4][2], qa[4][2];
#pragma unroll
      for (int r = 0; r < 4; ++r) ka[r][0] = ka[r][1] = qa[r][0] = qa[r][1] = 0.f;
#pragma unroll 4
      for (int kk = 0; kk < kGdnDim; ++kk) {
        const float2 kj = *reinterpret_cast<const float2*>(&S.kt[kk * kGdnChunk + 2 * lane]);
        const float4 k4 = *reinterpret_cast<const float4*>(&S.kt[kk * kGdnChunk + 4 * warp]);
        const float4 q4 = *reinterpret_cast<const float4*>(&S.qt[kk * kGdnChunk + 4 * warp]);
        const float kr[4] = {k4.x, k4.y, k4.z, k4.w}, qr[4] = {q4.x, q4.y, q4.z, q4.w};
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          ka[r][0] = fmaf(kr[r], kj.x, ka[r][0]);
          ka[r][1] = fmaf(kr[r], kj.y, ka[r][1]);
          qa[r][0] = fmaf(qr[r], kj.x, qa[r][0]);
          qa[r][1] = fmaf(qr[r], kj.y, qa[r][1]);
        }
      }
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const int t = 4 * warp + r;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          const int j = 2 * lane + c;
          const float dec = j <= t ? __expf(S.g[t] - S.g[j]) : 0.f;
          S.a[t * kGdnChunk + j] = j < t ? dec * ka[r][c] : 0.f;
          S.m[t * kGdnChunk + j] = dec * qa[r][c];
        }
      }
      if (tid < kGdnChunk) S.wk[tid] = __expf(S.g[kGdnChunk - 1] - S.g[tid]);
    }
    __syncthreads();
    // ---- U by forward substitution: thread c owns value column c ----
    if (tid < kGdnDim) {
      const int c = tid;
      float u[kGdnChunk];
#pragma unroll
      for (int t = 0; t < kGdnChunk; ++t) {
        float acc[4] = {S.v[t * kGdnDim + c], 0.f, 0.f, 0.f};
#pragma unroll
        for (int j = 0; j < t; ++j) acc[j & 3] = fmaf(-S.a[t * kGdnChunk + j], u[j], acc[j & 3]);
        u[t] = S.beta[t] * ((acc[0] + acc[1]) + (acc[2] + acc[3]));
        S.v[t * kGdnDim + c] = u[t];
      }
    }
    __syncthreads();
    // ---- O = diag(e^g) Q S0^T + M U, written for rows t < n ----
    {
      float o[4][4];
#pragma unroll
      for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int c = 0; c < 4; ++c) o[r][c] = qs[r][c];
#pragma unroll 4
      for (int j = 0; j < kGdnChunk; ++j) {
        const float4 u4 = *reinterpret_cast<const float4*>(&S.v[j * kGdnDim + 4 * lane]);
        const float uv[4] = {u4.x, u4.y, u4.z, u4.w};
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const float mr = S.m[(4 * warp + r) * kGdnChunk + j];
#pragma unroll
          for (int c = 0; c < 4; ++c) o[r][c] = fmaf(mr, uv[c], o[r][c]);
        }
      }
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const int t = 4 * warp + r;
        if (t < n) {
          uint2 pk;
          pk.x = pack_bf16x2(o[r][0], o[r][1]);
          pk.y = pack_bf16x2(o[r][2], o[r][3]);
          *reinterpret_cast<uint2*>(a.out + ((t0 + t) * a.heads + h) * kGdnDim + 4 * lane) = pk;
        }
      }
    }
    // ---- S^T = e^(g_C) S0^T + (diag(e^(g_C - g)) K)^T U: keys 4 kb .. +3, values 8 vb .. +7 ----
    {
      const int kb = tid >> 4, vb = tid & 15;
      const float gc = __expf(S.g[kGdnChunk - 1]);
      float acc[4][8];
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const float4* sp = reinterpret_cast<const float4*>(&S.st[(4 * kb + r) * kGdnDim + 8 * vb]);
        const float4 x = sp[0], y = sp[1];
        acc[r][0] = gc * x.x; acc[r][1] = gc * x.y; acc[r][2] = gc * x.z; acc[r][3] = gc * x.w;
        acc[r][4] = gc * y.x; acc[r][5] = gc * y.y; acc[r][6] = gc * y.z; acc[r][7] = gc * y.w;
      }
#pragma unroll 4
      for (int t = 0; t < kGdnChunk; ++t) {
        const float w = S.wk[t];
        const float4* up = reinterpret_cast<const float4*>(&S.v[t * kGdnDim + 8 * vb]);
        const float4 x = up[0], y = up[1];
        const float uv[8] = {x.x, x.y, x.z, x.w, y.x, y.y, y.z, y.w};
        const float4 k4 = *reinterpret_cast<const float4*>(&S.k[t * kGdnKStride + 4 * kb]);
        const float kw[4] = {w * k4.x, w * k4.y, w * k4.z, w * k4.w};
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const float kr = kw[r];
#pragma unroll
          for (int c = 0; c < 8; ++c) acc[r][c] = fmaf(kr, uv[c], acc[r][c]);
        }
      }
      // each thread rewrites only the entries it read; every read of whole rows of S0^T (for
      // K S0^T and Q S0^T) came before the barrier after A and M
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        float4* sp = reinterpret_cast<float4*>(&S.st[(4 * kb + r) * kGdnDim + 8 * vb]);
        sp[0] = make_float4(acc[r][0], acc[r][1], acc[r][2], acc[r][3]);
        sp[1] = make_float4(acc[r][4], acc[r][5], acc[r][6], acc[r][7]);
      }
    }
    __syncthreads();
  }
  if (a.final_state != nullptr) {
    float* fs = a.final_state + (static_cast<int64_t>(s) * a.heads + h) * kGdnDim * kGdnDim;
    for (int e = tid; e < kGdnDim * kGdnDim; e += kGdnThreads) {
      const int vv = e / kGdnDim, kk = e % kGdnDim;
      fs[e] = S.st[kk * kGdnDim + vv];
    }
  }
}

}  // namespace qsa
