// qsa_gdn.cuh -- the Gated DeltaNet linear-attention layer (the three of every four
// token-mixing layers around QSA), chunked, with the products on the tensor cores.
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
//     S_C = e^(g_C) S0 + (diag(e^(g_C - g)) U)^T K
// One CTA of 512 threads per (sequence, head) walks the sequence's chunks of 64 tokens in
// order.  The products K S0^T, Q S0^T, K K^T, Q K^T, M U and the state update run as warp
// tensor-core MMAs (m16n8k8, TF32 operands, fp32 accumulation); the forward substitution runs
// on the FMA pipes.  q, k and v arrive in bf16, which TF32 holds exactly, so K K^T and Q K^T
// are exact.  The fp32 operands that reach the state, S0 in K S0^T and e^(g_C - g) U in the
// update, are split into a TF32 head and a TF32 remainder (two MMAs, about fp32 accuracy);
// Q S0^T and M U feed only the bf16 output and take one rounded operand.  The state stays
// fp32 in shared memory.  log_alpha is clamped at -87 (alpha below about 1.6e-38 acts as a
// full reset), which keeps the differences g_t - g_j finite.

#pragma once

#include "qsa_common.cuh"

namespace qsa {

constexpr int kGdnDim = 128;      // d_k = d_v
constexpr int kGdnChunk = 64;
constexpr int kGdnThreads = 512;
constexpr float kGdnMinLogAlpha = -87.f;
// Row strides (floats).  An MMA operand fragment reads 8 rows x 4 columns (A, or B stored
// n-major) or 4 rows x 8 columns (B stored k-major): strides of 4 and 8 modulo 32 banks make
// each of the two conflict-free, and keep every row 16-byte aligned.
constexpr int kGdnLdA = kGdnDim + 4;      // 132: rows read as 8 x 4
constexpr int kGdnLdB = kGdnDim + 8;      // 136: rows read as 4 x 8
constexpr int kGdnLdT = kGdnChunk + 4;    // 68: A and M

struct GdnSmem {
  float st[kGdnDim * kGdnLdA];          // S[v][d], fp32
  float kr[kGdnChunk * kGdnLdA];        // K[t][d]
  float x[kGdnChunk * kGdnLdB];         // Q[t][d] (stride 132), then K[t][d] again (stride 136)
  float v[kGdnChunk * kGdnLdB];         // V, then V - diag(e^g) K S0^T, then U (fp32)
  float a[kGdnChunk * kGdnLdT];         // A (strictly lower), fp32
  float m[kGdnChunk * kGdnLdT];         // M (lower, diagonal included), TF32-rounded
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

// x rounded to TF32 (nearest, ties away), as a 32-bit operand register
__device__ __forceinline__ uint32_t gdn_tf32(float x) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
  return r;
}

// c += a b for one 16 x 8 x 8 tile: a (16 x 8, row-major fragment), b (8 x 8, column
// fragment), c (16 x 8) fp32.  Fragment of lane l, with gq = l / 4 and tq = l % 4:
//   a = {A[gq][tq], A[gq+8][tq], A[gq][tq+4], A[gq+8][tq+4]},  b = {B[tq][gq], B[tq+4][gq]},
//   c = {C[gq][2tq], C[gq][2tq+1], C[gq+8][2tq], C[gq+8][2tq+1]}.
__device__ __forceinline__ void gdn_mma(float* c, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// eight bf16 (one 16-byte word) to fp32 at dst (16-byte aligned)
__device__ __forceinline__ void gdn_store8(float* dst, uint4 w) {
  float4* d = reinterpret_cast<float4*>(dst);
  d[0] = make_float4(bf16_bits_to_float(w.x & 0xffffu), bf16_bits_to_float(w.x >> 16),
                     bf16_bits_to_float(w.y & 0xffffu), bf16_bits_to_float(w.y >> 16));
  d[1] = make_float4(bf16_bits_to_float(w.z & 0xffffu), bf16_bits_to_float(w.z >> 16),
                     bf16_bits_to_float(w.w & 0xffffu), bf16_bits_to_float(w.w >> 16));
}

// Rows t < n of the chunk starting at token t0 into shared memory (fp32); rows n..63 are
// zero with beta 0 and log gate 0, so they neither write nor decay the state.
__device__ __forceinline__ void gdn_load_chunk(const GdnArgs& a, GdnSmem& S, int h, int64_t t0,
                                               int n) {
  const int tid = threadIdx.x;
  // 1,024 groups of 8 values per matrix; lanes take consecutive groups of a row
  for (int e = tid; e < kGdnChunk * (kGdnDim / 8); e += kGdnThreads) {
    const int t = e / (kGdnDim / 8), d0 = (e % (kGdnDim / 8)) * 8;
    uint4 rq = make_uint4(0u, 0u, 0u, 0u), rk = rq, rv = rq;
    if (t < n) {
      const int64_t off = ((t0 + t) * a.heads + h) * kGdnDim + d0;
      rq = *reinterpret_cast<const uint4*>(a.q + off);
      rk = *reinterpret_cast<const uint4*>(a.k + off);
      rv = *reinterpret_cast<const uint4*>(a.v + off);
    }
    gdn_store8(&S.x[t * kGdnLdA + d0], rq);
    gdn_store8(&S.kr[t * kGdnLdA + d0], rk);
    gdn_store8(&S.v[t * kGdnLdB + d0], rv);
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
  const int gq = lane >> 2, tq = lane & 3;
  const int h = blockIdx.x, s = blockIdx.y;
  const int64_t t_begin = a.cu[s], t_end = a.cu[s + 1];
  for (int e = tid; e < kGdnDim * kGdnLdA; e += kGdnThreads) S.st[e] = 0.f;
  __syncthreads();
  // this warp's tiles: chunk rows r0 .. r0+15 with value columns c0 + 8 cb (K S0^T, Q S0^T,
  // O) and key columns j0 + 8 jb (A, M); for the state, value rows v0 .. v0+15 with key
  // columns d0 + 8 cb
  const int r0 = 16 * (warp & 3), c0 = 32 * (warp >> 2), j0 = 16 * (warp >> 2);
  const int v0 = 16 * (warp & 7), d0 = 64 * (warp >> 3);
  const int ta = r0 + gq, tb = ta + 8;   // the two chunk rows of this lane's fragments
  for (int64_t t0 = t_begin; t0 < t_end; t0 += kGdnChunk) {
    const int n = static_cast<int>(t_end - t0 < kGdnChunk ? t_end - t0 : kGdnChunk);
    gdn_load_chunk(a, S, h, t0, n);
    __syncthreads();
    // ---- K S0^T (S0 split in two TF32 parts), Q S0^T, K K^T and Q K^T in one pass over d ----
    float qs[4][4];
    {
      float w[4][4], am[2][4], mm[2][4];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int e = 0; e < 4; ++e) w[i][e] = qs[i][e] = 0.f;
#pragma unroll
      for (int i = 0; i < 2; ++i)
#pragma unroll
        for (int e = 0; e < 4; ++e) am[i][e] = mm[i][e] = 0.f;
#pragma unroll 2
      for (int k0 = 0; k0 < kGdnDim; k0 += 8) {
        const float* kp = &S.kr[ta * kGdnLdA + k0 + tq];
        const float* qp = &S.x[ta * kGdnLdA + k0 + tq];
        const uint32_t ak[4] = {__float_as_uint(kp[0]), __float_as_uint(kp[8 * kGdnLdA]),
                                __float_as_uint(kp[4]), __float_as_uint(kp[8 * kGdnLdA + 4])};
        const uint32_t aq[4] = {__float_as_uint(qp[0]), __float_as_uint(qp[8 * kGdnLdA]),
                                __float_as_uint(qp[4]), __float_as_uint(qp[8 * kGdnLdA + 4])};
#pragma unroll
        for (int cb = 0; cb < 4; ++cb) {
          // B[d][v] = S0[v][d]
          const float* sp = &S.st[(c0 + 8 * cb + gq) * kGdnLdA + k0 + tq];
          const float s0 = sp[0], s1 = sp[4];
          const uint32_t h0 = gdn_tf32(s0), h1 = gdn_tf32(s1);
          const uint32_t l0 = gdn_tf32(s0 - __uint_as_float(h0));
          const uint32_t l1 = gdn_tf32(s1 - __uint_as_float(h1));
          gdn_mma(w[cb], ak, h0, h1);
          gdn_mma(w[cb], ak, l0, l1);
          gdn_mma(qs[cb], aq, h0, h1);
        }
#pragma unroll
        for (int jb = 0; jb < 2; ++jb) {
          // B[d][j] = K[j][d]
          const float* bp = &S.kr[(j0 + 8 * jb + gq) * kGdnLdA + k0 + tq];
          const uint32_t b0 = __float_as_uint(bp[0]), b1 = __float_as_uint(bp[4]);
          gdn_mma(am[jb], ak, b0, b1);
          gdn_mma(mm[jb], aq, b0, b1);
        }
      }
      const float ea = __expf(S.g[ta]), eb = __expf(S.g[tb]);
#pragma unroll
      for (int cb = 0; cb < 4; ++cb) {
        const int vc = c0 + 8 * cb + 2 * tq;
        float2* pa = reinterpret_cast<float2*>(&S.v[ta * kGdnLdB + vc]);
        float2* pb = reinterpret_cast<float2*>(&S.v[tb * kGdnLdB + vc]);
        float2 xa = *pa, xb = *pb;
        xa.x -= ea * w[cb][0];
        xa.y -= ea * w[cb][1];
        xb.x -= eb * w[cb][2];
        xb.y -= eb * w[cb][3];
        *pa = xa;
        *pb = xb;
        qs[cb][0] *= ea;
        qs[cb][1] *= ea;
        qs[cb][2] *= eb;
        qs[cb][3] *= eb;
      }
#pragma unroll
      for (int jb = 0; jb < 2; ++jb) {
        const int jc = j0 + 8 * jb + 2 * tq;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int t = e < 2 ? ta : tb, j = jc + (e & 1);
          const float dec = j <= t ? __expf(S.g[t] - S.g[j]) : 0.f;
          S.a[t * kGdnLdT + j] = j < t ? dec * am[jb][e] : 0.f;
          S.m[t * kGdnLdT + j] = __uint_as_float(gdn_tf32(dec * mm[jb][e]));
        }
      }
      if (tid < kGdnChunk) S.wk[tid] = __expf(S.g[kGdnChunk - 1] - S.g[tid]);
    }
    __syncthreads();
    if (tid < kGdnDim) {
      // ---- U by forward substitution: thread c owns value column c ----
      const int c = tid;
      float u[kGdnChunk];
#pragma unroll
      for (int t = 0; t < kGdnChunk; ++t) {
        float acc[4] = {S.v[t * kGdnLdB + c], 0.f, 0.f, 0.f};
#pragma unroll
        for (int j = 0; j < t; ++j) acc[j & 3] = fmaf(-S.a[t * kGdnLdT + j], u[j], acc[j & 3]);
        u[t] = S.beta[t] * ((acc[0] + acc[1]) + (acc[2] + acc[3]));
        S.v[t * kGdnLdB + c] = u[t];
      }
    } else {
      // meanwhile the other warps copy K to the stride the state update reads (Q is done)
      for (int e = tid - kGdnDim; e < kGdnChunk * (kGdnDim / 4); e += kGdnThreads - kGdnDim) {
        const int t = e / (kGdnDim / 4), d = (e % (kGdnDim / 4)) * 4;
        *reinterpret_cast<float4*>(&S.x[t * kGdnLdB + d]) =
            *reinterpret_cast<const float4*>(&S.kr[t * kGdnLdA + d]);
      }
    }
    __syncthreads();
    // ---- O = diag(e^g) Q S0^T + M U on the same tiles as Q S0^T; M is zero above row r0+15 ----
    for (int k0 = 0; k0 < r0 + 16; k0 += 8) {
      const float* mp = &S.m[ta * kGdnLdT + k0 + tq];
      const uint32_t amt[4] = {__float_as_uint(mp[0]), __float_as_uint(mp[8 * kGdnLdT]),
                               __float_as_uint(mp[4]), __float_as_uint(mp[8 * kGdnLdT + 4])};
#pragma unroll
      for (int cb = 0; cb < 4; ++cb) {
        // B[j][v] = U[j][v]
        const float* up = &S.v[(k0 + tq) * kGdnLdB + c0 + 8 * cb + gq];
        gdn_mma(qs[cb], amt, gdn_tf32(up[0]), gdn_tf32(up[4 * kGdnLdB]));
      }
    }
#pragma unroll
    for (int cb = 0; cb < 4; ++cb) {
      const int vc = c0 + 8 * cb + 2 * tq;
      if (ta < n)
        *reinterpret_cast<uint32_t*>(a.out + ((t0 + ta) * a.heads + h) * kGdnDim + vc) =
            pack_bf16x2(qs[cb][0], qs[cb][1]);
      if (tb < n)
        *reinterpret_cast<uint32_t*>(a.out + ((t0 + tb) * a.heads + h) * kGdnDim + vc) =
            pack_bf16x2(qs[cb][2], qs[cb][3]);
    }
    // ---- S = e^(g_C) S0 + (diag(e^(g_C - g)) U)^T K, the scaled U split in two TF32 parts ----
    {
      const float gc = __expf(S.g[kGdnChunk - 1]);
      float acc[8][4];
#pragma unroll
      for (int cb = 0; cb < 8; ++cb) {
        const int dc = d0 + 8 * cb + 2 * tq;
        const float2 xa = *reinterpret_cast<const float2*>(&S.st[(v0 + gq) * kGdnLdA + dc]);
        const float2 xb = *reinterpret_cast<const float2*>(&S.st[(v0 + gq + 8) * kGdnLdA + dc]);
        acc[cb][0] = gc * xa.x;
        acc[cb][1] = gc * xa.y;
        acc[cb][2] = gc * xb.x;
        acc[cb][3] = gc * xb.y;
      }
#pragma unroll 2
      for (int k0 = 0; k0 < kGdnChunk; k0 += 8) {
        // A[v][t] = e^(g_C - g_t) U[t][v]
        const float w0 = S.wk[k0 + tq], w1 = S.wk[k0 + tq + 4];
        const float* up = &S.v[(k0 + tq) * kGdnLdB + v0 + gq];
        const float f[4] = {w0 * up[0], w0 * up[8], w1 * up[4 * kGdnLdB], w1 * up[4 * kGdnLdB + 8]};
        uint32_t hi[4], lo[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          hi[i] = gdn_tf32(f[i]);
          lo[i] = gdn_tf32(f[i] - __uint_as_float(hi[i]));
        }
#pragma unroll
        for (int cb = 0; cb < 8; ++cb) {
          // B[t][d] = K[t][d]
          const float* kp = &S.x[(k0 + tq) * kGdnLdB + d0 + 8 * cb + gq];
          const uint32_t b0 = __float_as_uint(kp[0]), b1 = __float_as_uint(kp[4 * kGdnLdB]);
          gdn_mma(acc[cb], hi, b0, b1);
          gdn_mma(acc[cb], lo, b0, b1);
        }
      }
      // each thread rewrites only the entries it read; every read of S0 (K S0^T, Q S0^T) came
      // before the barrier after A and M
#pragma unroll
      for (int cb = 0; cb < 8; ++cb) {
        const int dc = d0 + 8 * cb + 2 * tq;
        *reinterpret_cast<float2*>(&S.st[(v0 + gq) * kGdnLdA + dc]) = make_float2(acc[cb][0], acc[cb][1]);
        *reinterpret_cast<float2*>(&S.st[(v0 + gq + 8) * kGdnLdA + dc]) = make_float2(acc[cb][2], acc[cb][3]);
      }
    }
    __syncthreads();
  }
  if (a.final_state != nullptr) {
    float* fs = a.final_state + (static_cast<int64_t>(s) * a.heads + h) * kGdnDim * kGdnDim;
    for (int e = tid; e < kGdnDim * kGdnDim; e += kGdnThreads)
      fs[e] = S.st[(e / kGdnDim) * kGdnLdA + e % kGdnDim];
  }
}

}  // namespace qsa
