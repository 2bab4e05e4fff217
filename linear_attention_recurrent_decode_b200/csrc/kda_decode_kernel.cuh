// kda_decode_kernel.cuh -- sm_100a kernels of the recurrent KDA decode step.
//
// One CTA of 128 threads owns one (sequence n, value head h, 32-column value
// tile) of the fp32 state S[K][V] (V contiguous).  The CTA
//   1. reads slot_idx[n] and issues every 128-bit load of its K x 32 state tile
//      at once (8 KiB..32 KiB in flight per CTA, all straight into registers:
//      the tile is touched exactly once, so shared-memory staging would only
//      add a copy; the grid holds enough CTAs per SM to keep HBM busy);
//   2. for each token: decays its rows by exp(g), forms the two reductions
//      S'^T k and S'^T q over K (in-thread over its rows, warp shuffles across
//      the 4 row groups of a warp, shared memory across the 4 warps), the
//      correction u = beta (v - S'^T k), the rank-1 write S += k u^T and the
//      readout o = scale (S'^T q + (q.k) u), which equals scale S^T q of the
//      updated state without a second pass over it;
//   3. writes the tile back to the same slot once, after the last token.
// The state therefore crosses HBM exactly once in each direction per call.
//
// The gated variant launches the V/32 tiles of one (n, h) as a thread-block
// cluster: each CTA pushes its partial sum of o^2 into every peer's shared
// memory (DSMEM) and a cluster barrier completes the RMS over V; the norm,
// weight and sigmoid gate are applied before the bf16 store.
//
// No tensor cores: the step is a chain of mat-vec products with O(1) flops
// per state byte, far below any tensor-core ridge point; the roofline is HBM.
//
// Sources (pages by title): vLLM #57585 "Tune recurrent KDA launch
// configuration on SM90" (BF16 inputs, FP32 recurrent state, K = V = 128;
// Triton grid over (N*HV, V tiles)); FlashInfer #4562 "feat(cake_kda): add
// optimized H12 packed decode across SM100 family" (value tiles per head,
// 128-thread CTAs, state rows staged per tile; state_indices and scale as
// launch arguments); b12x #249 "feat(gdn): add direct single-token KDA decode"
// (decode then gated RMS norm of the output).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace kda {

constexpr int kThreads = 128;            // 4 warps
constexpr int kWarps = kThreads / 32;
constexpr int kBV = 32;                  // value columns per CTA
constexpr int kColQuads = kBV / 4;       // float4 column groups per row segment (8)
constexpr int kRowGroups = 32 / kColQuads;  // row groups per warp (4)
constexpr int kMaxClusterTiles = 8;      // portable cluster size bound

struct Params {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  const __nv_bfloat16* v;
  const float* g;
  const float* beta;
  float* state;
  const int32_t* slot_idx;
  __nv_bfloat16* out;
  const __nv_bfloat16* gate;         // gated variant only
  const __nv_bfloat16* norm_weight;  // gated variant only
  int64_t T;
  int64_t HV;
  int64_t V;
  int32_t tiles;  // V / kBV
  float scale;
  float eps;
};

// ---------------------------------------------------------------- helpers
__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&p);
}

// NB bf16 values starting at p (16-byte aligned when NB >= 8, 8-byte when NB == 4),
// through the read-only path.  Returned as packed pairs.
template <int NB>
struct Bf16Row {
  uint32_t w[NB / 2];
};

template <int NB>
__device__ __forceinline__ Bf16Row<NB> load_bf16_row(const __nv_bfloat16* p) {
  Bf16Row<NB> r;
  if constexpr (NB % 8 == 0) {
#pragma unroll
    for (int i = 0; i < NB / 8; ++i) {
      uint4 x = __ldg(reinterpret_cast<const uint4*>(p) + i);
      r.w[4 * i + 0] = x.x; r.w[4 * i + 1] = x.y; r.w[4 * i + 2] = x.z; r.w[4 * i + 3] = x.w;
    }
  } else {
    static_assert(NB == 4, "row chunk of 4 or a multiple of 8 bf16 values");
    uint2 x = __ldg(reinterpret_cast<const uint2*>(p));
    r.w[0] = x.x; r.w[1] = x.y;
  }
  return r;
}

template <int NF>
__device__ __forceinline__ void load_f32_row(float (&d)[NF], const float* p) {
  static_assert(NF % 4 == 0, "multiple of 4 floats");
#pragma unroll
  for (int i = 0; i < NF / 4; ++i) {
    float4 x = __ldg(reinterpret_cast<const float4*>(p) + i);
    d[4 * i + 0] = x.x; d[4 * i + 1] = x.y; d[4 * i + 2] = x.z; d[4 * i + 3] = x.w;
  }
}

// Inputs of one token for one thread: its RPT key rows of q, k, g and its 4
// value columns of v (and of the gate z).
template <int RPT, bool GATED>
struct TokenIn {
  Bf16Row<RPT> q, k;
  float g[RPT];
  Bf16Row<4> v;
  Bf16Row<4> z;
  float beta;
};

template <int RPT, bool GATED>
__device__ __forceinline__ TokenIn<RPT, GATED> load_token(const Params& p, int64_t row_qk,
                                                          int64_t row_v, int64_t row_b) {
  TokenIn<RPT, GATED> in;
  in.q = load_bf16_row<RPT>(p.q + row_qk);
  in.k = load_bf16_row<RPT>(p.k + row_qk);
  load_f32_row<RPT>(in.g, p.g + row_qk);
  in.v = load_bf16_row<4>(p.v + row_v);
  if constexpr (GATED) in.z = load_bf16_row<4>(p.gate + row_v);
  in.beta = __ldg(p.beta + row_b);
  return in;
}

// ---------------------------------------------------------------- cluster
__device__ __forceinline__ uint32_t smem_u32(const void* ptr) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(ptr));
}
__device__ __forceinline__ uint32_t cluster_map(uint32_t local_addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(local_addr), "r"(rank));
  return r;
}
__device__ __forceinline__ void cluster_store_f32(uint32_t cluster_addr, float x) {
  asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(cluster_addr), "f"(x) : "memory");
}
__device__ __forceinline__ void cluster_arrive_relaxed() {
  asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_arrive_release() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait_acquire() {
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// ---------------------------------------------------------------- kernel
// Thread layout inside the CTA (K x 32 tile, 128 threads):
//   warp w owns key rows [w*K/4, (w+1)*K/4); inside a warp, lane = rg*8 + cq
//   with row group rg in [0,4) and column quad cq in [0,8); the thread holds
//   rows r0 .. r0+RPT-1 (r0 = w*K/4 + rg*RPT, RPT = K/16) of columns
//   4cq .. 4cq+3 of the tile.  One warp-wide float4 load covers 4 rows x 128 B.
//
// MULTI = false is the T == 1 specialisation: no next-token prefetch registers.
//
// Resident CTAs per SM the register budget is capped for: at K = 128, T = 1
// seven CTAs (<= 72 registers a thread) put 1036 tiles in flight on 148 SMs,
// one wave for 32 sequences x 8 heads x 4 tiles.
template <int K, bool MULTI>
struct MinBlocks {
  static constexpr int value = MULTI ? (K >= 256 ? 2 : (K >= 128 ? 3 : 5)) : (K >= 256 ? 3 : (K >= 128 ? 7 : 8));
};

template <int K, bool GATED, bool MULTI>
__global__ void __launch_bounds__(kThreads, (MinBlocks<K, MULTI>::value))
kda_decode_kernel(const Params p) {
  constexpr int RPT = K / (kWarps * kRowGroups);
  static_assert(RPT * kWarps * kRowGroups == K && (RPT == 4 || RPT % 8 == 0), "K in {64,128,256}");

  __shared__ float4 red[2][kWarps][2 * kColQuads + 1];  // S'^T k | S'^T q | (q.k, -, -, -)
  __shared__ float nrm[2][kMaxClusterTiles];            // gated: per-tile sum of o^2

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int cq = lane & (kColQuads - 1);
  const int rg = lane / kColQuads;
  const int r0 = warp * (K / kWarps) + rg * RPT;

  const int64_t unit = blockIdx.x / p.tiles;  // n * HV + h
  const int tile = static_cast<int>(blockIdx.x - unit * p.tiles);
  const int64_t n = unit / p.HV;
  const int64_t h = unit - n * p.HV;
  const int64_t col = static_cast<int64_t>(tile) * kBV + cq * 4;
  const bool writer = (warp == 0) && (rg == 0);  // 8 lanes store the tile's 32 outputs

  const int32_t slot = __ldg(p.slot_idx + n);

  if (slot < 0) {  // inactive (padding) row: zero output, pool untouched
    if (writer) {
      for (int64_t t = 0; t < p.T; ++t) {
        const int64_t row_v = ((n * p.T + t) * p.HV + h) * p.V + col;
        *reinterpret_cast<uint2*>(p.out + row_v) = make_uint2(0u, 0u);
      }
    }
    return;  // uniform over the cluster: every tile of this (n, h) sees the same slot
  }

  if constexpr (GATED) cluster_arrive_relaxed();  // peers must be running before DSMEM writes

  // Token 0 inputs and the whole state tile, issued back to back.
  const int64_t qk_stride_t = p.HV * K;
  const int64_t v_stride_t = p.HV * p.V;
  int64_t row_qk = (n * p.T * p.HV + h) * K + r0;
  int64_t row_v = (n * p.T * p.HV + h) * p.V + col;
  int64_t row_b = n * p.T * p.HV + h;
  TokenIn<RPT, GATED> cur = load_token<RPT, GATED>(p, row_qk, row_v, row_b);

  float4* const sp = reinterpret_cast<float4*>(
      p.state + ((static_cast<int64_t>(slot) * p.HV + h) * K + r0) * p.V + col);
  float4 s[RPT];
#pragma unroll
  for (int i = 0; i < RPT; ++i) s[i] = sp[i * (p.V / 4)];

  float wgt[4] = {0.f, 0.f, 0.f, 0.f};
  if constexpr (GATED) {
    Bf16Row<4> w = load_bf16_row<4>(p.norm_weight + col);
    wgt[0] = bf16lo(w.w[0]); wgt[1] = bf16hi(w.w[0]); wgt[2] = bf16lo(w.w[1]); wgt[3] = bf16hi(w.w[1]);
  }

  for (int64_t t = 0; t < p.T; ++t) {
    const int buf = static_cast<int>(t & 1);
    TokenIn<RPT, GATED> nxt;
    if constexpr (MULTI) {
      if (t + 1 < p.T) nxt = load_token<RPT, GATED>(p, row_qk + qk_stride_t, row_v + v_stride_t, row_b + p.HV);
    }

    // decay, partial reductions over this thread's rows
    float pk[4] = {0.f, 0.f, 0.f, 0.f}, pq[4] = {0.f, 0.f, 0.f, 0.f}, qk = 0.f;
#pragma unroll
    for (int i = 0; i < RPT; ++i) {
      const float qi = (i & 1) ? bf16hi(cur.q.w[i >> 1]) : bf16lo(cur.q.w[i >> 1]);
      const float ki = (i & 1) ? bf16hi(cur.k.w[i >> 1]) : bf16lo(cur.k.w[i >> 1]);
      const float d = expf(cur.g[i]);
      s[i].x *= d; s[i].y *= d; s[i].z *= d; s[i].w *= d;
      pk[0] = fmaf(s[i].x, ki, pk[0]); pk[1] = fmaf(s[i].y, ki, pk[1]);
      pk[2] = fmaf(s[i].z, ki, pk[2]); pk[3] = fmaf(s[i].w, ki, pk[3]);
      pq[0] = fmaf(s[i].x, qi, pq[0]); pq[1] = fmaf(s[i].y, qi, pq[1]);
      pq[2] = fmaf(s[i].z, qi, pq[2]); pq[3] = fmaf(s[i].w, qi, pq[3]);
      qk = fmaf(qi, ki, qk);
    }
    // across the 4 row groups of the warp
#pragma unroll
    for (int m = kColQuads; m < 32; m <<= 1) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        pk[j] += __shfl_xor_sync(0xffffffffu, pk[j], m);
        pq[j] += __shfl_xor_sync(0xffffffffu, pq[j], m);
      }
      qk += __shfl_xor_sync(0xffffffffu, qk, m);
    }
    // across the 4 warps
    if (rg == 0) {
      red[buf][warp][cq] = make_float4(pk[0], pk[1], pk[2], pk[3]);
      red[buf][warp][kColQuads + cq] = make_float4(pq[0], pq[1], pq[2], pq[3]);
      if (cq == 0) red[buf][warp][2 * kColQuads] = make_float4(qk, 0.f, 0.f, 0.f);
    }
    __syncthreads();
    float rk[4] = {0.f, 0.f, 0.f, 0.f}, rq[4] = {0.f, 0.f, 0.f, 0.f}, qkt = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      const float4 a = red[buf][w][cq];
      const float4 b = red[buf][w][kColQuads + cq];
      rk[0] += a.x; rk[1] += a.y; rk[2] += a.z; rk[3] += a.w;
      rq[0] += b.x; rq[1] += b.y; rq[2] += b.z; rq[3] += b.w;
      qkt += red[buf][w][2 * kColQuads].x;
    }
    // correction, rank-1 write, readout
    const float vv[4] = {bf16lo(cur.v.w[0]), bf16hi(cur.v.w[0]), bf16lo(cur.v.w[1]), bf16hi(cur.v.w[1])};
    float u[4], o[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      u[j] = cur.beta * (vv[j] - rk[j]);
      o[j] = p.scale * fmaf(qkt, u[j], rq[j]);
    }
#pragma unroll
    for (int i = 0; i < RPT; ++i) {
      const float ki = (i & 1) ? bf16hi(cur.k.w[i >> 1]) : bf16lo(cur.k.w[i >> 1]);
      s[i].x = fmaf(ki, u[0], s[i].x); s[i].y = fmaf(ki, u[1], s[i].y);
      s[i].z = fmaf(ki, u[2], s[i].z); s[i].w = fmaf(ki, u[3], s[i].w);
    }

    if constexpr (GATED) {
      // per-tile sum of o^2 (lanes 0..7 of warp 0 hold the tile's 32 outputs)
      float ss = 0.f;
      if (writer) {
        ss = o[0] * o[0] + o[1] * o[1] + o[2] * o[2] + o[3] * o[3];
#pragma unroll
        for (int m = 1; m < kColQuads; m <<= 1) ss += __shfl_xor_sync(0x000000ffu, ss, m);
      }
      if (t == 0) cluster_wait_acquire();  // pairs with the relaxed arrive at kernel start
      if (writer && lane < p.tiles) {
        cluster_store_f32(cluster_map(smem_u32(&nrm[buf][tile]), static_cast<uint32_t>(lane)), ss);
      }
      cluster_arrive_release();
      cluster_wait_acquire();
      if (writer) {
        float tot = 0.f;
        for (int r = 0; r < p.tiles; ++r) tot += nrm[buf][r];
        const float inv = rsqrtf(tot / static_cast<float>(p.V) + p.eps);
        const float zz[4] = {bf16lo(cur.z.w[0]), bf16hi(cur.z.w[0]), bf16lo(cur.z.w[1]), bf16hi(cur.z.w[1])};
#pragma unroll
        for (int j = 0; j < 4; ++j) o[j] = o[j] * inv * wgt[j] * (1.0f / (1.0f + expf(-zz[j])));
      }
    }
    if (writer) {
      *reinterpret_cast<uint2*>(p.out + row_v) = make_uint2(pack_bf16x2(o[0], o[1]), pack_bf16x2(o[2], o[3]));
    }

    row_qk += qk_stride_t;
    row_v += v_stride_t;
    row_b += p.HV;
    if constexpr (MULTI) {
      if (t + 1 < p.T) cur = nxt;
    } else {
      break;  // T == 1
    }
  }

#pragma unroll
  for (int i = 0; i < RPT; ++i) sp[i * (p.V / 4)] = s[i];
}

}  // namespace kda
