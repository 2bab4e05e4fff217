// kda_prefill_kernel.cuh -- sm_100a kernels of the chunked KDA prefill.
//
// The same recurrence as the decode step, taken over long token runs: per
// sequence n and value head h, for t = 0 .. T-1,
//   S <- Diag(exp(g_t)) S;  u_t = beta_t (v_t - S^T k_t);  S <- S + k_t u_t^T;
//   o_t = scale S^T q_t.
// Tokens are grouped in chunks of C = 64 and the recurrence is regrouped into
// the WY / UT chunk form (vLLM #57585 "Tune recurrent KDA launch configuration
// on SM90", Details: FlashInfer's fused KDA prefill path on Blackwell is the
// related work the page names).  Inside a chunk, with Gamma_t = sum_{s<=t} g_s
// (per key channel, the cumulative log-decay from the chunk start) and S0 the
// state at the chunk start:
//   Kt_t = k_t * exp(Gamma_t)            (decayed keys)
//   Qt_t = q_t * exp(Gamma_t)            (decayed queries)
//   Kh_t = k_t * exp(Gamma_C - Gamma_t)  (keys decayed to the chunk end)
//   M[t][s] = sum_i k_t,i k_s,i exp(Gamma_t,i - Gamma_s,i)   (s < t)
//   P[t][s] = sum_i q_t,i k_s,i exp(Gamma_t,i - Gamma_s,i)   (s <= t)
// the corrections solve the unit lower-triangular system
//   u_t + beta_t sum_{s<t} M[t][s] u_s = beta_t (v_t - S0^T Kt_t),
// i.e. U = Ut - W S0 with [W | Ut] = (I + diag(beta) M)^-1 diag(beta) [Kt | V],
// and then
//   O   = scale (Qt S0 + P U),
//   S_C = Diag(exp(Gamma_C)) S0 + Kh^T U.
// This equals the token-by-token recurrence in exact arithmetic.
//
// Three kernels:
//   1. kda_prefill_chunk_kernel (one CTA per (n, h, chunk), all chunks at
//      once): Gamma in fp64, the decay factors, M and P, the substitution for
//      W and Ut; writes them to the workspace.
//   2. kda_prefill_state_kernel (one CTA per (n, h, 8/16/32-column value tile),
//      chunks in order): the state chain U = Ut - W S0, S_C = D S0 + Kh^T U,
//      keeping S in shared memory; writes each chunk's start state and U to the
//      workspace and the final state back to the pool slot.
//   3. kda_prefill_output_kernel (one CTA per (n, h, chunk)): O = scale (Qt S0
//      + P U) on the tensor cores (tcgen05), bf16 output.
//
// Numerics.  exp(Gamma_t - Gamma_s) is never formed by dividing decays: the
// chunk kernel factors it as exp(Gamma_t - Gamma_r) exp(Gamma_r - Gamma_s)
// around the chunk's middle token r, which keeps both factors in fp32 range
// whenever every key channel decays by at most e^80 between r and any token
// of the chunk; a chunk outside that bound (a decay of more than e^-2.5 per
// token on some channel, sustained over half a chunk) takes a slower exact
// path that forms every pair's exponential directly.  Gamma is summed in fp64
// and each exponential is taken from the fp64 difference, so the long-range
// decays keep fp32 accuracy (a cumulative sum in fp32 would lose up to
// 64 ulp of |Gamma|).  All other arithmetic is fp32, except the output
// products, whose bf16-pair operands carry 16 significant bits (see kernel 3).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace kdap {

constexpr int kC = 64;        // tokens per chunk
constexpr int kK = 128;       // key dimension (the kernels are written for K = V = 128)
constexpr int kV = 128;       // value dimension
constexpr float kSafeExp = 80.f;  // |Gamma_t - Gamma_r| bound of the factored path

struct Params {
  const __nv_bfloat16* q;  // [N, T, HV, K]
  const __nv_bfloat16* k;  // [N, T, HV, K]
  const __nv_bfloat16* v;  // [N, T, HV, V]
  const float* g;          // [N, T, HV, K]
  const float* beta;       // [N, T, HV]
  float* state;            // [num_slots, HV, K, V]
  const int32_t* slot_idx; // [N]
  __nv_bfloat16* out;      // [N, T, HV, V]
  float* ws;               // workspace (see Workspace)
  int64_t T;
  int64_t HV;
  int32_t nchunks;         // ceil(T / C)
  float scale;
};

// Workspace layout: a 256-byte header (word 0: the error word, see
// wait_bounded), then one fp32 record per (n, h, chunk).
struct Workspace {
  static constexpr int64_t kHeaderFloats = 64;
  static constexpr int64_t kWt = 0;                   // W^T  [K][C]
  static constexpr int64_t kKh = kWt + kK * kC;       // Kh   [C][K]
  static constexpr int64_t kUt = kKh + kC * kK;       // Ut   [C][V]   (the V part of the solve)
  // The output operands, as bf16 hi and lo planes in the canonical K-major
  // layout (see put_pair): rows x K-dimension of each MMA operand.
  static constexpr int64_t kQ = kUt + kC * kV;        // Qt   [C rows][K]  (decayed queries)
  static constexpr int64_t kP = kQ + kC * kK;         // P    [C rows][C]  (zero for s > t)
  static constexpr int64_t kDc = kP + kC * kC;        // exp(Gamma_C) [K]  (fp32)
  static constexpr int64_t kS0 = kDc + kK;            // S0^T [V rows][K]  (chunk-start state)
  static constexpr int64_t kU = kS0 + kK * kV;        // U^T  [V rows][C]
  static constexpr int64_t kFloats = kU + kC * kV;    // per record
  static __host__ __device__ int64_t record(int64_t unit, int64_t chunk, int32_t nchunks) {
    return kHeaderFloats + (unit * nchunks + chunk) * kFloats;
  }
};

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------- output-operand tiles
// The output kernel's four MMA operands (S0^T, Qt, U^T, P) are written by the
// kernels that compute them straight into their workspace regions in the
// tensor cores' shared-memory layout, each as a bf16 hi plane followed by a
// bf16 lo plane (x = hi + lo, 16 significant bits; the same bytes as fp32),
// so that the output kernel moves them into shared memory with bulk copies.
// Offset, in bytes, of element (row r, k) of a K-major bf16 tile with kd
// elements along K (canonical layout, no swizzle).
__host__ __device__ constexpr uint32_t kmajor_off(int r, int k, int kd) {
  return static_cast<uint32_t>((r / 8) * (kd / 8) * 128 + (k / 8) * 128 + (r % 8) * 16 + (k % 8) * 2);
}
// The hi and lo bf16 halves of eight fp32 values, packed for one 16-byte store each.
__device__ __forceinline__ void split8(const float (&x)[8], uint4& hi, uint4& lo) {
  uint32_t h[4], l[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const __nv_bfloat162 hh = __floats2bfloat162_rn(x[2 * i], x[2 * i + 1]);
    const float2 hf = __bfloat1622float2(hh);
    const __nv_bfloat162 ll = __floats2bfloat162_rn(x[2 * i] - hf.x, x[2 * i + 1] - hf.y);
    h[i] = *reinterpret_cast<const uint32_t*>(&hh);
    l[i] = *reinterpret_cast<const uint32_t*>(&ll);
  }
  hi = make_uint4(h[0], h[1], h[2], h[3]);
  lo = make_uint4(l[0], l[1], l[2], l[3]);
}

// Element (r, c) of an fp32 operand tile as its bf16 pair: hi = bf16(x) into
// the hi plane at the canonical offset, lo = bf16(x - hi) at the same offset
// of the lo plane, `plane_bytes` after it (the same split as split8).
__device__ __forceinline__ void put_pair(unsigned char* hi_plane, int plane_bytes, int r, int c, int kd, float x) {
  const __nv_bfloat16 h = __float2bfloat16_rn(x);
  const __nv_bfloat16 l = __float2bfloat16_rn(x - __bfloat162float(h));
  const uint32_t off = kmajor_off(r, c, kd);
  *reinterpret_cast<__nv_bfloat16*>(hi_plane + off) = h;
  *reinterpret_cast<__nv_bfloat16*>(hi_plane + plane_bytes + off) = l;
}

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_addr(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// exp(x) for an fp64 argument, to fp32 accuracy: expf of the fp32 part times
// (1 + the remainder), the remainder being below half an fp32 ulp of x.
__device__ __forceinline__ float exp_of(double x) {
  const float hi = static_cast<float>(x);
  const float lo = static_cast<float>(x - static_cast<double>(hi));
  return expf(hi) * (1.0f + lo);
}

// ---------------------------------------------------------------- kernel 1
// Shared memory of the chunk kernel (dynamic; about 200 KB).
// Rows of the transposed factor buffers are padded to 68 floats: the stores
// from consecutive key channels then spread over the banks (4-way instead of
// 32-way), and every row still starts on a 16-byte boundary for the float4
// reads of the Gram products.
constexpr int kCP = kC + 4;
struct ChunkSmem {
  double gam[kC][kK];               // Gamma_t, the cumulative log-decay from the chunk start; 64 KB
  float kt[kC][kK];                 // Kt = k exp(Gamma_t) [t][i]; the solve reads its columns
  float at[kK][kCP];                // k_t exp(Gamma_t - Gamma_r) [i][t]
  float aq[kK][kCP];                // q_t exp(Gamma_t - Gamma_r) [i][t]
  float bk[kK][kCP];                // k_s exp(Gamma_r - Gamma_s) [i][s]
  float L[kC][kC];                  // beta_t M[t][s] (s < t), zero elsewhere
  float e_ref[kK];                  // exp(Gamma_r) per channel (factored path)
  float e_end_ref[kK];              // exp(Gamma_C - Gamma_r) per channel (factored path)
  float beta[kC];
  int exact;                        // some channel is outside the factored path's range
};
// The raw bf16 inputs are staged over `at` .. `bk` before the factors are formed.
struct ChunkRaw {
  __nv_bfloat16 q[kC][kK];
  __nv_bfloat16 k[kC][kK];
  __nv_bfloat16 v[kC][kV];
};
static_assert(sizeof(ChunkRaw) <= 3 * kK * kCP * sizeof(float), "raw inputs fit over the factor buffers");

constexpr int kChunkThreads = 512;

__global__ void __launch_bounds__(kChunkThreads, 1) kda_prefill_chunk_kernel(const Params p) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  ChunkSmem& sm = *reinterpret_cast<ChunkSmem*>(smem_raw);
  ChunkRaw& raw = *reinterpret_cast<ChunkRaw*>(&sm.at[0][0]);

  const int tid = threadIdx.x;
  const int64_t unit = blockIdx.x / p.nchunks;  // n * HV + h
  const int32_t chunk = static_cast<int32_t>(blockIdx.x - unit * p.nchunks);
  const int64_t n = unit / p.HV;
  const int64_t h = unit - n * p.HV;
  const int64_t t0 = static_cast<int64_t>(chunk) * kC;
  const int tc = static_cast<int>(p.T - t0 < kC ? p.T - t0 : kC);  // tokens in this chunk
  if (__ldg(p.slot_idx + n) < 0) return;  // inactive row: nothing to prepare

  // ---- 1. stage q, k, v (bf16) and beta; g goes straight to fp64 cumulative sums
  for (int c = tid; c < kC * (kK / 8); c += kChunkThreads) {  // q and k: 16 pieces of 16 B per row
    const int t = c / (kK / 8), pc = c % (kK / 8);
    if (t < tc) {
      const int64_t row = ((n * p.T + t0 + t) * p.HV + h);
      cp_async16(&raw.q[t][pc * 8], p.q + row * kK + pc * 8);
      cp_async16(&raw.k[t][pc * 8], p.k + row * kK + pc * 8);
      cp_async16(&raw.v[t][pc * 8], p.v + row * kV + pc * 8);
    } else {
      *reinterpret_cast<uint4*>(&raw.q[t][pc * 8]) = make_uint4(0, 0, 0, 0);
      *reinterpret_cast<uint4*>(&raw.k[t][pc * 8]) = make_uint4(0, 0, 0, 0);
      *reinterpret_cast<uint4*>(&raw.v[t][pc * 8]) = make_uint4(0, 0, 0, 0);
    }
  }
  // g goes through the kt buffer (free until step 2): 32 pieces of 16 B per
  // row; rows past the chunk's end are zeros (those tokens do not decay)
  for (int c = tid; c < kC * (kK / 4); c += kChunkThreads) {
    const int t = c / (kK / 4), pc = c % (kK / 4);
    if (t < tc) cp_async16(&sm.kt[t][pc * 4], p.g + ((n * p.T + t0 + t) * p.HV + h) * kK + pc * 4);
    else *reinterpret_cast<float4*>(&sm.kt[t][pc * 4]) = make_float4(0.f, 0.f, 0.f, 0.f);
  }
  cp_async_commit();
  if (tid < kC) sm.beta[tid] = tid < tc ? __ldg(p.beta + (n * p.T + t0 + tid) * p.HV + h) : 0.f;
  if (tid == 0) sm.exact = 0;
  cp_async_wait<0>();
  __syncthreads();

  // Gamma per key channel, summed in fp64 in token order: four threads per
  // channel each sum a quarter of the chunk, then each adds the totals of the
  // quarters before its own.  The reference token r is the chunk's middle.
  constexpr int kRef = kC / 2 - 1;
  static_assert(kChunkThreads % kK == 0 && kC % (kChunkThreads / kK) == 0, "whole quarters per channel");
  constexpr int kQT = kC / (kChunkThreads / kK);  // tokens per thread
  const int ci = tid % kK, cq = tid / kK;          // this thread's channel and part of the chunk
  {
    double acc = 0.0;
#pragma unroll
    for (int t = cq * kQT; t < (cq + 1) * kQT; ++t) {
      acc += static_cast<double>(sm.kt[t][ci]);
      sm.gam[t][ci] = acc;
    }
  }
  __syncthreads();
  {
    double off = 0.0;
    for (int q = 0; q < cq; ++q) off += sm.gam[(q + 1) * kQT - 1][ci];
    __syncthreads();  // every part's total is read before any part adds its offset
    if (cq > 0) {
#pragma unroll
      for (int t = cq * kQT; t < (cq + 1) * kQT; ++t) sm.gam[t][ci] += off;
    }
  }
  __syncthreads();
  double gam_end = 0.0;  // per channel (the threads of the first part)
  {
    const double gam_ref = sm.gam[kRef][ci];
    double worst = 0.0;
#pragma unroll
    for (int t = cq * kQT; t < (cq + 1) * kQT; ++t) worst = fmax(worst, fabs(sm.gam[t][ci] - gam_ref));
    // the factored path also forms exp(Gamma_r) and exp(Gamma_C - Gamma_r): keep
    // them normal fp32 numbers
    if (worst > kSafeExp || gam_ref < -kSafeExp) atomicOr(&sm.exact, 1);
    if (cq == 0) {
      gam_end = sm.gam[kC - 1][ci];
      sm.e_ref[ci] = exp_of(gam_ref);
      sm.e_end_ref[ci] = exp_of(gam_end - gam_ref);
    }
  }
  __syncthreads();
  const bool exact = sm.exact != 0;

  // ---- 2. per-token decays: the workspace's Kh and Qt, the solve's Kt, and on
  // the factored path the factors around the reference token r, from two
  // exponentials per element (exp(+-(Gamma_t - Gamma_r))) and the channel's
  // exp(Gamma_r), exp(Gamma_C - Gamma_r).
  float* const rec = p.ws + Workspace::record(unit, chunk, p.nchunks);
  unsigned char* const q_pl = reinterpret_cast<unsigned char*>(rec + Workspace::kQ);  // Qt planes
  unsigned char* const p_pl = reinterpret_cast<unsigned char*>(rec + Workspace::kP);  // P planes
  constexpr int kQPlane = kC * kK * 2, kPPlane = kC * kC * 2;
  if (tid < kK) rec[Workspace::kDc + tid] = exp_of(gam_end);
  constexpr int kPer = kC * kK / kChunkThreads;  // elements per thread
  if (!exact) {
    // The factors go through registers: the raw inputs they are made from live
    // in the buffers they are written to.
    float fa[kPer], fq[kPer], fb[kPer];
    // each thread keeps its channel ci
    const double g_ref = sm.gam[kRef][ci];
    const float er = sm.e_ref[ci], eer = sm.e_end_ref[ci];
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
      const int e = tid + j * kChunkThreads;  // consecutive threads, consecutive channels
      const int t = e / kK, i = ci;
      const double d = sm.gam[t][i] - g_ref;
      const float up = exp_of(d);      // exp(Gamma_t - Gamma_r), in [e^-80, e^80] on this path
      const float down = __frcp_rn(up);  // exp(Gamma_r - Gamma_t), correctly rounded reciprocal
      const float kv = __bfloat162float(raw.k[t][i]);
      const float qv = __bfloat162float(raw.q[t][i]);
      fa[j] = kv * up;
      fq[j] = qv * up;
      fb[j] = kv * down;
      sm.kt[t][i] = fa[j] * er;                                          // k exp(Gamma_t)
      rec[Workspace::kKh + t * kK + i] = fb[j] * eer;                    // k exp(Gamma_C - Gamma_t)
      put_pair(q_pl, kQPlane, t, i, kK, fq[j] * er);                     // q exp(Gamma_t)
    }
    __syncthreads();
    // The solve needs v, which the factors overwrite: move it into the Gamma
    // buffer (no longer needed on this path) as fp32 [t][j].
    float* const vf = reinterpret_cast<float*>(&sm.gam[0][0]);
    for (int e = tid; e < kC * kV; e += kChunkThreads) vf[e] = __bfloat162float(raw.v[e / kV][e % kV]);
    __syncthreads();
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
      const int e = tid + j * kChunkThreads;
      const int t = e / kK, i = e % kK;
      sm.at[i][t] = fa[j];
      sm.aq[i][t] = fq[j];
      sm.bk[i][t] = fb[j];
    }
    __syncthreads();
    // ---- 3. M and P in 4 x 4 tiles of (t, s): the 136 tiles on or below the
    // diagonal go to the first 136 threads (whole warps past them skip the
    // loop), the 120 tiles above it are zeros written by the next 120 threads.
    constexpr int kTb = kC / 4;                           // tile rows (16)
    constexpr int kLower = kTb * (kTb + 1) / 2;          // 136
    int tb, sb;
    if (tid < kLower) {  // tid -> (tb, sb) with sb <= tb, row by row
      tb = static_cast<int>((sqrtf(8.f * tid + 1.f) - 1.f) * 0.5f);
      while ((tb + 1) * (tb + 2) / 2 <= tid) ++tb;
      while (tb * (tb + 1) / 2 > tid) --tb;
      sb = tid - tb * (tb + 1) / 2;
      float2 m[4][2], pp[4][2];  // pairs of s
#pragma unroll
      for (int a = 0; a < 4; ++a) m[a][0] = m[a][1] = pp[a][0] = pp[a][1] = make_float2(0.f, 0.f);
#pragma unroll 4
      for (int i = 0; i < kK; ++i) {
        const float4 A = *reinterpret_cast<const float4*>(&sm.at[i][tb * 4]);
        const float4 Q = *reinterpret_cast<const float4*>(&sm.aq[i][tb * 4]);
        const float4 B = *reinterpret_cast<const float4*>(&sm.bk[i][sb * 4]);
        const float av[4] = {A.x, A.y, A.z, A.w}, qv[4] = {Q.x, Q.y, Q.z, Q.w};
        const float2 b01 = make_float2(B.x, B.y), b23 = make_float2(B.z, B.w);
#pragma unroll
        for (int a = 0; a < 4; ++a) {
          m[a][0] = __ffma2_rn(make_float2(av[a], av[a]), b01, m[a][0]);
          m[a][1] = __ffma2_rn(make_float2(av[a], av[a]), b23, m[a][1]);
          pp[a][0] = __ffma2_rn(make_float2(qv[a], qv[a]), b01, pp[a][0]);
          pp[a][1] = __ffma2_rn(make_float2(qv[a], qv[a]), b23, pp[a][1]);
        }
      }
#pragma unroll
      for (int a = 0; a < 4; ++a) {
        const int t = tb * 4 + a;
        const float mv[4] = {m[a][0].x, m[a][0].y, m[a][1].x, m[a][1].y};
        const float pv[4] = {pp[a][0].x, pp[a][0].y, pp[a][1].x, pp[a][1].y};
#pragma unroll
        for (int b = 0; b < 4; ++b) {
          const int s = sb * 4 + b;
          sm.L[t][s] = (s < t) ? sm.beta[t] * mv[b] : 0.f;
          put_pair(p_pl, kPPlane, t, s, kC, (s <= t) ? pv[b] : 0.f);
        }
      }
    } else if (tid < kLower + kTb * (kTb - 1) / 2) {  // the 120 tiles above the diagonal: zeros
      // k -> (r, c) with c < r in the strict lower triangle, mirrored to (tb, sb) = (c, r)
      const int k = tid - kLower;
      int r = static_cast<int>((sqrtf(8.f * k + 1.f) + 1.f) * 0.5f);
      while (r * (r - 1) / 2 > k) --r;
      while ((r + 1) * r / 2 <= k) ++r;
      tb = k - r * (r - 1) / 2;
      sb = r;
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) {
          sm.L[tb * 4 + a][sb * 4 + b] = 0.f;
          put_pair(p_pl, kPPlane, tb * 4 + a, sb * 4 + b, kC, 0.f);
        }
    }
  } else {
    // Exact path (rare: decays beyond e^80 within half a chunk): every
    // exponential from its own fp64 Gamma difference.
    for (int e = tid; e < kC * kK; e += kChunkThreads) {
      const int t = e / kK, i = e % kK;
      const double gt = sm.gam[t][i];
      const float kv = __bfloat162float(raw.k[t][i]);
      const float dt = exp_of(gt);
      sm.kt[t][i] = kv * dt;                                                   // k exp(Gamma_t)
      rec[Workspace::kKh + t * kK + i] = kv * exp_of(sm.gam[kC - 1][i] - gt);  // k exp(Gamma_C - Gamma_t)
      put_pair(q_pl, kQPlane, t, i, kK, __bfloat162float(raw.q[t][i]) * dt);   // q exp(Gamma_t)
    }
    for (int e = tid; e < kC * kC; e += kChunkThreads) {
      const int t = e / kC, s = e % kC;
      float mv = 0.f, pv = 0.f;
      if (s <= t) {
        for (int i = 0; i < kK; ++i) {
          const float w = __bfloat162float(raw.k[s][i]) * exp_of(sm.gam[t][i] - sm.gam[s][i]);
          mv = fmaf(__bfloat162float(raw.k[t][i]), w, mv);
          pv = fmaf(__bfloat162float(raw.q[t][i]), w, pv);
        }
      }
      sm.L[t][s] = (s < t) ? sm.beta[t] * mv : 0.f;
      put_pair(p_pl, kPPlane, t, s, kC, (s <= t) ? pv : 0.f);
    }
    __syncthreads();
    float* const vf = reinterpret_cast<float*>(&sm.gam[0][0]);
    // gam is dead after the loop above; v moves there as on the fast path
    float vtmp[kC * kV / kChunkThreads];
#pragma unroll
    for (int j = 0; j < kC * kV / kChunkThreads; ++j) {
      const int e = tid + j * kChunkThreads;
      vtmp[j] = __bfloat162float(raw.v[e / kV][e % kV]);
    }
    __syncthreads();
#pragma unroll
    for (int j = 0; j < kC * kV / kChunkThreads; ++j) vf[tid + j * kChunkThreads] = vtmp[j];
  }
  __syncthreads();

  // ---- 4. forward substitution: X[t] = beta_t R[t] - sum_{s<t} L[t][s] X[s],
  // R = [Kt | V]; thread j < K + V owns column j (j < K: W, else Ut).  Blocks of 16
  // tokens: the earlier blocks' contribution is a small product over solved
  // rows kept in shared memory (rolled over the blocks), the in-block
  // triangle is unrolled; the same arithmetic as a row-by-row solve with a
  // quarter of the code (the kernel was stalling on instruction fetch).
  if (tid < kK + kV) {
    constexpr int kB = 16;                                   // tokens per block
    constexpr int kCols = kK + kV;                           // solve columns
    const int j = tid;
    const float* const vf = reinterpret_cast<const float*>(&sm.gam[0][0]);
    float* const X = &sm.at[0][0];                           // [kC][kCols] solved rows (the factors are dead)
    static_assert(kC * kCols <= 3 * kK * kCP, "solved rows fit over the factor buffers");
    for (int b = 0; b < kC / kB; ++b) {
      const int t0b = b * kB;
      float xb[kB];
#pragma unroll
      for (int t = 0; t < kB; ++t)
        xb[t] = sm.beta[t0b + t] * (j < kK ? sm.kt[t0b + t][j] : vf[(t0b + t) * kV + (j - kK)]);
      for (int pb = 0; pb < b; ++pb) {  // earlier blocks
        const int s0 = pb * kB;
        float2 xs[kB / 2];
#pragma unroll
        for (int u = 0; u < kB / 2; ++u) xs[u] = make_float2(X[(s0 + 2 * u) * kCols + j], X[(s0 + 2 * u + 1) * kCols + j]);
#pragma unroll
        for (int t = 0; t < kB; ++t) {
          float2 acc = make_float2(0.f, 0.f);
#pragma unroll
          for (int q4 = 0; q4 < kB / 4; ++q4) {
            const float4 l = *reinterpret_cast<const float4*>(&sm.L[t0b + t][s0 + 4 * q4]);
            acc = __ffma2_rn(make_float2(l.x, l.y), xs[2 * q4], acc);
            acc = __ffma2_rn(make_float2(l.z, l.w), xs[2 * q4 + 1], acc);
          }
          xb[t] -= acc.x + acc.y;
        }
      }
#pragma unroll
      for (int t = 1; t < kB; ++t) {  // in-block triangle
#pragma unroll
        for (int s2 = 0; s2 < t; ++s2) xb[t] = fmaf(-sm.L[t0b + t][t0b + s2], xb[s2], xb[t]);
      }
#pragma unroll
      for (int t = 0; t < kB; ++t) X[(t0b + t) * kCols + j] = xb[t];
      if (j < kK) {
        float* const wt = rec + Workspace::kWt + j * kC + t0b;  // W^T row j
#pragma unroll
        for (int t = 0; t < kB; t += 4) *reinterpret_cast<float4*>(wt + t) = make_float4(xb[t], xb[t + 1], xb[t + 2], xb[t + 3]);
      } else {
        float* const ut = rec + Workspace::kUt + (j - kK);
#pragma unroll
        for (int t = 0; t < kB; ++t) ut[(t0b + t) * kV] = xb[t];
      }
    }
  }
}

// ---------------------------------------------------------------- kernel 2
// One CTA of NT threads per (n, h, BV-column value tile) walks the chunks in
// order with its K x BV state tile in shared memory.  Per chunk:
// U = Ut - W S0 (W S split over quarters of K) and S = D S0 + Kh^T U (Kh^T U
// split over parts of the chunk for narrow tiles), packed fp32x2 FMAs, the
// partials summed in a fixed order.
// Staging: the next chunk's operands are copied (cp.async) while the current
// one is processed.  Narrow tiles (8, 16 columns) double-buffer all of them.
// Wide tiles keep one buffer each for W^T and Kh (64 KB together), refilled
// for the next chunk as soon as the product that reads it is done (W^T after
// W S, Kh after Kh^T U) -- their longer chunk steps leave each copy time to
// land -- which is what lets a 64-column tile's buffers fit one SM.  The two
// products' partial sums share their bytes (one is dead while the other is in
// use).  Every CTA reads the
// chunk's 64 KB of W^T and Kh whatever its width, so the launch takes the
// narrowest tile whose CTAs fit one per SM in one wave, else 64-column tiles
// of 512 threads (see state_tile_width).
constexpr int kCU = kC + 4;  // padded rows of the transposed partial buffers

template <int BV, int NT>
struct StateCfg {
  static_assert((NT == 256 && (BV == 8 || BV == 16 || BV == 32)) || (NT == 512 && (BV == 32 || BV == 64)),
                "tile widths 8, 16, 32 (256 threads) and 32, 64 (512 threads)");
  static constexpr int kJW = 64 * BV / NT;   // W S: columns per thread (thread: K quarter, 4 tokens)
  static constexpr int kNJ = BV / kJW;       //       column groups
  static constexpr int kJW2 = BV == 8 ? 4 : 8;  // Kh^T U: columns per thread (thread: 2 key rows)
  static constexpr int kNG2 = BV / kJW2;        //         column groups
  static constexpr int kCS = NT / (64 * kNG2);  //         parts of the chunk
  static_assert(64 * kNG2 * kCS == NT && kC % kCS == 0, "Kh^T U covers the tile once");
  static constexpr int kUW = 64 * BV / NT;   // U: columns per thread (thread: one token)
  static constexpr int kRT = NT / kK;        // S update: threads per key row
  static constexpr int kSW = BV / kRT;       //           columns per thread
  static_assert(kJW % 2 == 0 && kSW % 4 == 0, "packed pairs and float4 rows");
  static constexpr int kPart = 4 * BV * kCU > kCS * BV * (kK + 4) ? 4 * BV * kCU : kCS * BV * (kK + 4);
  static constexpr bool kDB = BV <= 16;      // W^T and Kh double-buffered
  static constexpr int kNB = kDB ? 2 : 1;
  struct UBuf {
    float ut[kC][BV];  // this tile's columns of Ut
    float dc[kK];      // exp(Gamma_C)
  };
  struct Smem {
    float wt[kNB][kK][kC];  // W^T of the current chunk (and of the next: see kDB)
    float kh[kNB][kC][kK];  // Kh, likewise
    UBuf ub[2];
    float s[kK][BV];        // state tile
    float u[kC][BV + 4];    // U of the current chunk, [t][j]
    float part[kPart];      // (W S) partials [4][BV][kCU], then (Kh^T U) partials [kCS][BV][kK + 4]
  };
};

template <int NT>
__device__ __forceinline__ void stage_wt(float (&wt)[kK][kC], const float* rec, int tid) {
  for (int c = tid; c < (kK * kC) / 4; c += NT) cp_async16(&wt[0][0] + 4 * c, rec + Workspace::kWt + 4 * c);
}
template <int NT>
__device__ __forceinline__ void stage_kh(float (&kh)[kC][kK], const float* rec, int tid) {
  for (int c = tid; c < (kC * kK) / 4; c += NT) cp_async16(&kh[0][0] + 4 * c, rec + Workspace::kKh + 4 * c);
}
template <int BV, int NT>
__device__ __forceinline__ void stage_ub(typename StateCfg<BV, NT>::UBuf& b, const float* rec, int col0, int tid) {
  for (int c = tid; c < kC * (BV / 4); c += NT) {
    const int t = c / (BV / 4), pc = c % (BV / 4);
    cp_async16(&b.ut[t][pc * 4], rec + Workspace::kUt + t * kV + col0 + pc * 4);
  }
  for (int c = tid; c < kK / 4; c += NT) cp_async16(&b.dc[4 * c], rec + Workspace::kDc + 4 * c);
}

__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }
__device__ __forceinline__ float2 splat(float x) { return make_float2(x, x); }

template <int BV, int NT>
__global__ void __launch_bounds__(NT, 1) kda_prefill_state_kernel(const Params p) {
  using Cfg = StateCfg<BV, NT>;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  typename Cfg::Smem& sm = *reinterpret_cast<typename Cfg::Smem*>(smem_raw);
  constexpr int kTiles = kV / BV;
  const int tid = threadIdx.x;
  const int64_t unit = blockIdx.x / kTiles;
  const int tile = static_cast<int>(blockIdx.x - unit * kTiles);
  const int col0 = tile * BV;
  const int64_t n = unit / p.HV;
  const int64_t h = unit - n * p.HV;
  const int32_t slot = __ldg(p.slot_idx + n);
  if (slot < 0) return;

  float* const blk = p.state + (static_cast<int64_t>(slot) * p.HV + h) * kK * kV;
  for (int c = tid; c < kK * (BV / 4); c += NT) {  // initial state tile
    const int i = c / (BV / 4), pc = c % (BV / 4);
    cp_async16(&sm.s[i][pc * 4], blk + i * kV + col0 + pc * 4);
  }
  {
    const float* const rec0 = p.ws + Workspace::record(unit, 0, p.nchunks);
    stage_wt<NT>(sm.wt[0], rec0, tid);
    stage_kh<NT>(sm.kh[0], rec0, tid);
    stage_ub<BV, NT>(sm.ub[0], rec0, col0, tid);
  }
  cp_async_commit();

  // W S: thread (quarter of K, 4 tokens, kJW columns)
  const int a_t = (tid % 16) * 4, a_j = ((tid / 16) % Cfg::kNJ) * Cfg::kJW, a_q = tid / (16 * Cfg::kNJ);
  // U: thread (token, kUW columns)
  const int u_t = tid % 64, u_j = (tid / 64) * Cfg::kUW;
  // Kh^T U: thread (2 key rows, kJW2 columns, part of the chunk)
  const int b_i = (tid % 64) * 2, b_j = ((tid / 64) % Cfg::kNG2) * Cfg::kJW2, b_h = tid / (64 * Cfg::kNG2);
  // S update: thread (key row, kSW columns)
  const int s_i = tid / Cfg::kRT, s_j = (tid % Cfg::kRT) * Cfg::kSW;
  float (*const pw)[BV][kCU] = reinterpret_cast<float (*)[BV][kCU]>(sm.part);
  float (*const ps)[BV][kK + 4] = reinterpret_cast<float (*)[BV][kK + 4]>(sm.part);

  for (int32_t c = 0; c < p.nchunks; ++c) {
    const int cb = c & 1;
    const bool more = c + 1 < p.nchunks;
    float* const rec = p.ws + Workspace::record(unit, c, p.nchunks);
    const float* const rec_next = p.ws + Workspace::record(unit, more ? c + 1 : c, p.nchunks);
    constexpr bool kDB = Cfg::kDB;
    const int wb = kDB ? cb : 0;  // this chunk's W^T and Kh buffers
    if (more) {
      stage_ub<BV, NT>(sm.ub[cb ^ 1], rec_next, col0, tid);
      if constexpr (kDB) {
        stage_wt<NT>(sm.wt[cb ^ 1], rec_next, tid);
        stage_kh<NT>(sm.kh[cb ^ 1], rec_next, tid);
      }
      cp_async_commit();
    }
    // This chunk's operands: with double buffers all of them, the next chunk's
    // copies in flight; with single ones W^T, Ut and exp(Gamma_C) (all of
    // chunk 0 at the start), this chunk's Kh and the next Ut in flight.
    if (kDB || c == 0) {
      if (more) cp_async_wait<1>(); else cp_async_wait<0>();
    } else {
      if (more) cp_async_wait<2>(); else cp_async_wait<1>();
    }
    __syncthreads();
    const typename Cfg::UBuf& ub = sm.ub[cb];
    const float (&wt)[kK][kC] = sm.wt[wb];
    const float (&kh)[kC][kK] = sm.kh[wb];

    // chunk-start state to the workspace as the output MMA's S0^T operand
    // (rows: this tile's value columns; 8 key rows per 16-byte store)
    unsigned char* const s0_pl = reinterpret_cast<unsigned char*>(rec + Workspace::kS0);
    for (int e = tid; e < BV * (kK / 8); e += NT) {
      const int jl = e % BV, ig = e / BV;
      float x[8];
#pragma unroll
      for (int r = 0; r < 8; ++r) x[r] = sm.s[ig * 8 + r][jl];
      uint4 hi, lo;
      split8(x, hi, lo);
      const uint32_t off = kmajor_off(col0 + jl, ig * 8, kK);
      *reinterpret_cast<uint4*>(s0_pl + off) = hi;
      *reinterpret_cast<uint4*>(s0_pl + kK * kV * 2 + off) = lo;
    }

    {  // W S over one quarter of K
      float2 acc[4][Cfg::kJW / 2];
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int jj = 0; jj < Cfg::kJW / 2; ++jj) acc[a][jj] = splat(0.f);
      const int i_lo = a_q * (kK / 4);
#pragma unroll 4
      for (int i = i_lo; i < i_lo + kK / 4; ++i) {
        const float4 w = *reinterpret_cast<const float4*>(&wt[i][a_t]);
        float2 sv[Cfg::kJW / 2];
        if constexpr (Cfg::kJW % 4 == 0) {
#pragma unroll
          for (int q4 = 0; q4 < Cfg::kJW / 4; ++q4) {
            const float4 x = *reinterpret_cast<const float4*>(&sm.s[i][a_j + 4 * q4]);
            sv[2 * q4] = make_float2(x.x, x.y);
            sv[2 * q4 + 1] = make_float2(x.z, x.w);
          }
        } else {
          sv[0] = *reinterpret_cast<const float2*>(&sm.s[i][a_j]);
        }
        const float wv[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
          for (int jj = 0; jj < Cfg::kJW / 2; ++jj) acc[a][jj] = ffma2(splat(wv[a]), sv[jj], acc[a][jj]);
      }
#pragma unroll
      for (int jj = 0; jj < Cfg::kJW / 2; ++jj) {
        *reinterpret_cast<float4*>(&pw[a_q][a_j + 2 * jj][a_t]) =
            make_float4(acc[0][jj].x, acc[1][jj].x, acc[2][jj].x, acc[3][jj].x);
        *reinterpret_cast<float4*>(&pw[a_q][a_j + 2 * jj + 1][a_t]) =
            make_float4(acc[0][jj].y, acc[1][jj].y, acc[2][jj].y, acc[3][jj].y);
      }
    }
    __syncthreads();  // the partials are complete; W^T is free for the next chunk's
    if (!kDB && more) {
      stage_wt<NT>(sm.wt[0], rec_next, tid);
      cp_async_commit();
    }
    {  // U = Ut - W S, the quarters summed in a fixed order
#pragma unroll
      for (int jj = 0; jj < Cfg::kUW; ++jj) {
        const int j = u_j + jj;
        const float ws = (pw[0][j][u_t] + pw[1][j][u_t]) + (pw[2][j][u_t] + pw[3][j][u_t]);
        sm.u[u_t][j] = ub.ut[u_t][j] - ws;
      }
    }
    // This chunk's Kh (chunk 0's came with the first group); the copies
    // committed after it (the next Ut and W^T) stay in flight.
    if (!kDB && c > 0) {
      if (more) cp_async_wait<2>(); else cp_async_wait<0>();
    }
    __syncthreads();  // U is complete; the W S partials are dead
    {  // U to the workspace as the output MMA's U^T operand (8 tokens per 16-byte store)
      unsigned char* const u_pl = reinterpret_cast<unsigned char*>(rec + Workspace::kU);
      for (int e = tid; e < BV * (kC / 8); e += NT) {
        const int jl = e % BV, tg = e / BV;
        float x[8];
#pragma unroll
        for (int r = 0; r < 8; ++r) x[r] = sm.u[tg * 8 + r][jl];
        uint4 hi, lo;
        split8(x, hi, lo);
        const uint32_t off = kmajor_off(col0 + jl, tg * 8, kC);
        *reinterpret_cast<uint4*>(u_pl + off) = hi;
        *reinterpret_cast<uint4*>(u_pl + kC * kV * 2 + off) = lo;
      }
    }
    {  // Kh^T U over one part of the chunk
      float2 acc[2][Cfg::kJW2 / 2];
#pragma unroll
      for (int a = 0; a < 2; ++a)
#pragma unroll
        for (int jj = 0; jj < Cfg::kJW2 / 2; ++jj) acc[a][jj] = splat(0.f);
      const int t_lo = b_h * (kC / Cfg::kCS);
#pragma unroll 4
      for (int t = t_lo; t < t_lo + kC / Cfg::kCS; ++t) {
        const float2 kv = *reinterpret_cast<const float2*>(&kh[t][b_i]);
        float2 uv[Cfg::kJW2 / 2];
#pragma unroll
        for (int q4 = 0; q4 < Cfg::kJW2 / 4; ++q4) {
          const float4 x = *reinterpret_cast<const float4*>(&sm.u[t][b_j + 4 * q4]);
          uv[2 * q4] = make_float2(x.x, x.y);
          uv[2 * q4 + 1] = make_float2(x.z, x.w);
        }
#pragma unroll
        for (int jj = 0; jj < Cfg::kJW2 / 2; ++jj) {
          acc[0][jj] = ffma2(splat(kv.x), uv[jj], acc[0][jj]);
          acc[1][jj] = ffma2(splat(kv.y), uv[jj], acc[1][jj]);
        }
      }
#pragma unroll
      for (int a = 0; a < 2; ++a)
#pragma unroll
        for (int jj = 0; jj < Cfg::kJW2 / 2; ++jj) {
          ps[b_h][b_j + 2 * jj][b_i + a] = acc[a][jj].x;
          ps[b_h][b_j + 2 * jj + 1][b_i + a] = acc[a][jj].y;
        }
    }
    // S = D S + Kh^T U.  The decay is read before the barrier: after it no
    // thread reads this chunk's Ut buffer, which the next iteration refills.
    const float d = ub.dc[s_i];
    __syncthreads();  // the partials are complete; Kh is free for the next chunk's
    if (!kDB && more) {
      stage_kh<NT>(sm.kh[0], rec_next, tid);
      cp_async_commit();
    }
#pragma unroll
    for (int q4 = 0; q4 < Cfg::kSW / 4; ++q4) {
      const int j = s_j + 4 * q4;
      const float4 s0 = *reinterpret_cast<const float4*>(&sm.s[s_i][j]);
      float hs[4];
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) {
        float acc = ps[0][j + jj][s_i];
#pragma unroll
        for (int cs = 1; cs < Cfg::kCS; ++cs) acc += ps[cs][j + jj][s_i];
        hs[jj] = acc;
      }
      *reinterpret_cast<float4*>(&sm.s[s_i][j]) =
          make_float4(fmaf(d, s0.x, hs[0]), fmaf(d, s0.y, hs[1]), fmaf(d, s0.z, hs[2]), fmaf(d, s0.w, hs[3]));
    }
    // The next iteration's first barrier orders these writes of s before any
    // read, and the partial buffer's reuse by its W S after this update.
  }
  __syncthreads();
  for (int c = tid; c < kK * (BV / 4); c += NT) {
    const int i = c / (BV / 4), pc = c % (BV / 4);
    *reinterpret_cast<float4*>(blk + i * kV + col0 + pc * 4) = *reinterpret_cast<const float4*>(&sm.s[i][pc * 4]);
  }
}

// The state kernel's value-tile width for N * HV heads: the narrowest tile
// whose CTAs (one per SM) fit in one wave of `sms` SMs, else 64 columns (512
// threads a CTA), which needs the fewest waves.
__host__ __device__ constexpr int state_tile_width(int64_t heads, int sms) {
  return heads * (kV / 8) <= sms ? 8 : (heads * (kV / 16) <= sms ? 16 : (heads * (kV / 32) <= sms ? 32 : 64));
}
// Threads of the state kernel for a tile width.
__host__ __device__ constexpr int state_threads(int bv) { return bv >= 64 ? 512 : 256; }
template <int BV, int NT>
constexpr int kStateSmem = static_cast<int>(sizeof(typename StateCfg<BV, NT>::Smem));

// ---------------------------------------------------------------- kernel 3
// The chunk outputs on the tensor cores (tcgen05, kind::f16), transposed so
// that the value index is the MMA's M = 128:
//   O^T [V x C] = S0^T [V x K] . Qt^T [K x C]  +  U^T [V x C] . P^T [C x C].
// fp32 operands are split into bf16 pairs x = hi + lo (hi = bf16(x),
// lo = bf16(x - hi): 16 significant bits), and each product takes three MMAs
// (hi.hi + hi.lo + lo.hi; the dropped lo.lo term is 2^-18 relative), so the
// fp32 accumulation in tensor memory is accurate to about 2^-16 -- well inside
// the bf16 output rounding.  Operand tiles sit in shared memory in the
// canonical K-major layout without swizzle: 8-row x 16-byte core matrices, the
// two core matrices of one 16-element K step 128 bytes apart (the leading byte
// offset) and consecutive 8-row groups (K/8) * 128 bytes apart (the stride
// byte offset).  One thread issues the 36 MMAs and commits them to an
// mbarrier; every thread then reads its value column's 64 outputs back from
// tensor memory (tcgen05.ld, lane = value column).
namespace tc {

__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  // start address, leading and stride byte offsets in 16-byte units; the
  // SM100 descriptor version (1) at bit 46; no swizzle, base offset 0
  return static_cast<uint64_t>((addr >> 4) & 0x3FFFu) | (static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16) |
         (static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46);
}
// kind::f16 instruction descriptor: fp32 accumulator, bf16 A and B, both
// K-major, N >> 3 at bit 17, M >> 4 at bit 24.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(M >> 4) << 24);
}
__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate));
}
__device__ __forceinline__ void commit(uint64_t* mbar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_addr(mbar))
               : "memory");
}
__device__ __forceinline__ void fence_before_sync() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_after_sync() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void mbar_init(uint64_t* mbar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(mbar)), "r"(count) : "memory");
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* mbar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(mbar)), "r"(bytes) : "memory");
}
// Bulk copy (TMA unit) of `bytes` contiguous bytes, global -> this CTA's shared
// memory (both 16-byte aligned, bytes a multiple of 16), completing on `mbar`.
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* mbar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
               ::"r"(smem_addr(dst)), "l"(src), "r"(bytes), "r"(smem_addr(mbar))
               : "memory");
}
// Wait for phase `parity` of the mbarrier, giving up after `limit` polls
// (returns false then): the kernels never wait without bound.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* mbar, uint32_t parity, uint32_t limit) {
  for (uint32_t i = 0; i < limit; ++i) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(done)
        : "r"(smem_addr(mbar)), "r"(parity)
        : "memory");
    if (done) return true;
  }
  return false;
}
__device__ __forceinline__ void tmem_alloc(uint32_t* dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(dst)), "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
// 16 consecutive fp32 columns of this thread's lane.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

}  // namespace tc

constexpr int kOutThreads = 256;
constexpr uint32_t kOutTmemCols = 64;  // the fp32 accumulator, 128 lanes x C columns

struct OutSmem {
  alignas(1024) unsigned char a1h[kV * kK * 2];  // S0^T  [V rows][K]  bf16 hi
  alignas(1024) unsigned char a1l[kV * kK * 2];  //                      lo
  alignas(1024) unsigned char b1h[kC * kK * 2];  // Qt    [C rows][K]
  alignas(1024) unsigned char b1l[kC * kK * 2];
  alignas(1024) unsigned char a2h[kV * kC * 2];  // U^T   [V rows][C]
  alignas(1024) unsigned char a2l[kV * kC * 2];
  alignas(1024) unsigned char b2h[kC * kC * 2];  // P     [C rows][C]
  alignas(1024) unsigned char b2l[kC * kC * 2];
  uint64_t mbar_in;  // the operand copies
  uint64_t mbar;     // the MMAs
  uint32_t tmem;
};

__global__ void __launch_bounds__(kOutThreads, 1) kda_prefill_output_kernel(const Params p) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  OutSmem& sm = *reinterpret_cast<OutSmem*>(smem_raw);
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int64_t unit = blockIdx.x / p.nchunks;
  const int32_t chunk = static_cast<int32_t>(blockIdx.x - unit * p.nchunks);
  const int64_t n = unit / p.HV;
  const int64_t h = unit - n * p.HV;
  const int64_t t0 = static_cast<int64_t>(chunk) * kC;
  const int tc = static_cast<int>(p.T - t0 < kC ? p.T - t0 : kC);
  // epilogue: value column j = 32 (warp % 4) + lane, tokens of half (warp / 4)
  const int j = 32 * (warp % 4) + lane;
  const int half = warp / 4;
  if (__ldg(p.slot_idx + n) < 0) {  // inactive row: zero output
    for (int t = half * 32; t < half * 32 + 32 && t < tc; ++t)
      p.out[((n * p.T + t0 + t) * p.HV + h) * kV + j] = __float2bfloat16(0.f);
    return;
  }
  if (warp == 0) tc::tmem_alloc(&sm.tmem, kOutTmemCols);
  if (tid == 0) {
    tc::mbar_init(&sm.mbar_in, 1);
    tc::mbar_init(&sm.mbar, 1);
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();

  // ---- operand tiles: the producers left them in this layout, as bf16 hi and
  // lo planes; eight bulk copies bring them in (144 KB).
  const unsigned char* const rec =
      reinterpret_cast<const unsigned char*>(p.ws + Workspace::record(unit, chunk, p.nchunks));
  if (tid == 0) {
    constexpr uint32_t kA1 = kV * kK * 2, kB1 = kC * kK * 2, kA2 = kV * kC * 2, kB2 = kC * kC * 2;
    tc::mbar_arrive_expect_tx(&sm.mbar_in, 2 * (kA1 + kB1 + kA2 + kB2));
    const unsigned char* const s0 = rec + Workspace::kS0 * 4;
    const unsigned char* const qt = rec + Workspace::kQ * 4;
    const unsigned char* const ut = rec + Workspace::kU * 4;
    const unsigned char* const pp = rec + Workspace::kP * 4;
    tc::bulk_load(sm.a1h, s0, kA1, &sm.mbar_in);
    tc::bulk_load(sm.a1l, s0 + kA1, kA1, &sm.mbar_in);
    tc::bulk_load(sm.b1h, qt, kB1, &sm.mbar_in);
    tc::bulk_load(sm.b1l, qt + kB1, kB1, &sm.mbar_in);
    tc::bulk_load(sm.a2h, ut, kA2, &sm.mbar_in);
    tc::bulk_load(sm.a2l, ut + kA2, kA2, &sm.mbar_in);
    tc::bulk_load(sm.b2h, pp, kB2, &sm.mbar_in);
    tc::bulk_load(sm.b2l, pp + kB2, kB2, &sm.mbar_in);
  }
  // about 2^26 polls: seconds, against microseconds for the copies and MMAs
  const bool in_ok = __syncthreads_and(tc::mbar_wait_bounded(&sm.mbar_in, 0, 1u << 26));
  const uint32_t tmem = sm.tmem;

  if (tid == 0 && in_ok) {
    constexpr uint32_t idesc = tc::idesc_bf16(128, kC);
    const uint32_t a1h = smem_addr(sm.a1h), a1l = smem_addr(sm.a1l), b1h = smem_addr(sm.b1h),
                   b1l = smem_addr(sm.b1l), a2h = smem_addr(sm.a2h), a2l = smem_addr(sm.a2l),
                   b2h = smem_addr(sm.b2h), b2l = smem_addr(sm.b2l);
    constexpr uint32_t kLbo = 128;
    constexpr uint32_t kSbo1 = (kK / 8) * 128;  // K = 128 along the K dimension
    constexpr uint32_t kSbo2 = (kC / 8) * 128;  // K = 64
    uint32_t acc = 0;
#pragma unroll
    for (int st = 0; st < kK / 16; ++st) {
      const uint32_t off = st * 256;  // two core matrices per 16-element K step
      tc::mma_bf16(tmem, tc::smem_desc(a1h + off, kLbo, kSbo1), tc::smem_desc(b1h + off, kLbo, kSbo1), idesc, acc);
      acc = 1;
      tc::mma_bf16(tmem, tc::smem_desc(a1h + off, kLbo, kSbo1), tc::smem_desc(b1l + off, kLbo, kSbo1), idesc, 1);
      tc::mma_bf16(tmem, tc::smem_desc(a1l + off, kLbo, kSbo1), tc::smem_desc(b1h + off, kLbo, kSbo1), idesc, 1);
    }
#pragma unroll
    for (int st = 0; st < kC / 16; ++st) {
      const uint32_t off = st * 256;
      tc::mma_bf16(tmem, tc::smem_desc(a2h + off, kLbo, kSbo2), tc::smem_desc(b2h + off, kLbo, kSbo2), idesc, 1);
      tc::mma_bf16(tmem, tc::smem_desc(a2h + off, kLbo, kSbo2), tc::smem_desc(b2l + off, kLbo, kSbo2), idesc, 1);
      tc::mma_bf16(tmem, tc::smem_desc(a2l + off, kLbo, kSbo2), tc::smem_desc(b2h + off, kLbo, kSbo2), idesc, 1);
    }
    tc::commit(&sm.mbar);
  }
  const bool ok = in_ok && tc::mbar_wait_bounded(&sm.mbar, 0, 1u << 26);
  tc::fence_after_sync();
  if (ok) {
    // lane j of this warp's 32-lane slice; columns (tokens) of this warp's half
    const uint32_t taddr = tmem + (static_cast<uint32_t>(32 * (warp % 4)) << 16) + static_cast<uint32_t>(half * 32);
    float o[32];
    tc::tmem_ld16(taddr, *reinterpret_cast<float(*)[16]>(&o[0]));
    tc::tmem_ld16(taddr + 16, *reinterpret_cast<float(*)[16]>(&o[16]));
#pragma unroll
    for (int c = 0; c < 32; ++c) {
      const int t = half * 32 + c;
      if (t < tc) p.out[((n * p.T + t0 + t) * p.HV + h) * kV + j] = __float2bfloat16_rn(p.scale * o[c]);
    }
  } else if (tid == 0) {
    atomicExch(reinterpret_cast<int*>(p.ws), 1);  // the workspace header's error word
    if (!in_ok) tc::mbar_wait_bounded(&sm.mbar_in, 0, 1u << 26);  // copies still in flight
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 0) tc::tmem_dealloc(tmem, kOutTmemCols);
}

constexpr int kChunkSmem = static_cast<int>(sizeof(ChunkSmem));
constexpr int kOutSmem = static_cast<int>(sizeof(OutSmem));

}  // namespace kdap
