// kda_decode_kernel.cuh -- sm_100a kernels of the recurrent KDA decode step.
//
// One CTA of 128 threads owns one (sequence n, value head h, 32-column value
// tile) of the fp32 state S[K][V] (V contiguous).  The CTA
//   1. reads slot_idx[n] and issues every 128-bit load of its K x 32 state tile
//      at once (8..32 KiB in flight per CTA), straight into registers: the tile
//      is touched exactly once, so staging it in shared memory would only add
//      a copy (a bulk-TMA staging of the same tile measured no faster on B200);
//   2. for each token: decays its rows by exp(g), forms the two reductions
//      S'^T k and S'^T q over K (in-thread over its rows, a reduce-scatter of
//      warp shuffles across the 4 row groups of a warp, shared memory across
//      the 4 warps), the correction u = beta (v - S'^T k), the rank-1 write
//      S += k u^T and the readout o = scale (S'^T q + (q.k) u), which equals
//      scale S^T q of the updated state without a second pass over it;
//   3. writes the tile back to the same slot once, after the last token.
// The state therefore crosses HBM exactly once in each direction per call.
//
// All per-element arithmetic uses Blackwell's packed fp32x2 instructions
// (__fmul2_rn / __ffma2_rn / __fadd2_rn: two IEEE round-to-nearest lanes per
// instruction).  The kernel is a single wave at serving batch sizes, so every
// CTA computes at the same moment after its loads land: instruction count is
// on the critical path, and the packed forms halve it.
//
// Multi-token calls (T > 1) stage the next chunk of tokens' q, k, g, v, gate
// and beta in shared memory with cp.async, so the state tile is the only
// per-thread register payload.
//
// The gated variant launches the V/32 tiles of one (n, h) as a thread-block
// cluster: each CTA pushes its partial sum of o^2 into every peer's shared
// memory (DSMEM) and a cluster barrier completes the RMS over V; the norm,
// weight and sigmoid gate are applied before the bf16 store.
//
// Launch overlap: kernels are launched with programmatic stream
// serialization.  Every global access of a CTA comes after griddepcontrol.wait
// (all work earlier in the stream complete and visible), and a CTA lets the
// next kernel in the stream start launching once it is about to write its
// state back, so the next call's launch overlaps this call's stores.  The
// state is written with streaming (evict-first) stores: it is not read again
// before the next decode step.
//
// No tensor cores: the step is a chain of mat-vec products with O(1) flops
// per state byte, far below any tensor-core ridge point; the roofline is HBM.
//
// Sources (pages by title): vLLM #57585 "Tune recurrent KDA launch
// configuration on SM90" (BF16 inputs, FP32 recurrent state, K = V = 128;
// Triton grid over (N*HV, V tiles)); FlashInfer #4562 "feat(cake_kda): add
// optimized H12 packed decode across SM100 family" (value tiles per head,
// 128-thread CTAs, cp.async staging; state_indices and scale as launch
// arguments); b12x #249 "feat(gdn): add direct single-token KDA decode"
// (decode then gated RMS norm of the output).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace kda {

constexpr int kThreads = 128;               // 4 warps
constexpr int kWarps = kThreads / 32;
constexpr int kBV = 32;                     // value columns per CTA
constexpr int kColQuads = kBV / 4;          // float4 column groups per row segment (8)
constexpr int kRowGroups = 32 / kColQuads;  // row groups per warp (4)
constexpr int kMaxClusterTiles = 8;         // portable cluster size bound
constexpr int kTokenChunk = 8;              // tokens staged in shared memory at a time (T > 1)

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
__device__ __forceinline__ float bf16_at(const uint32_t* w, int i) {
  return (i & 1) ? bf16hi(w[i >> 1]) : bf16lo(w[i >> 1]);
}
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&p);
}
__device__ __forceinline__ float2 f2(float a) { return make_float2(a, a); }

// RPT consecutive bf16 values (RPT = 4: 8 bytes; RPT % 8 == 0: 16-byte chunks).
template <int RPT>
__device__ __forceinline__ void ld_bf16_rows(uint32_t (&w)[RPT / 2], const __nv_bfloat16* p) {
  if constexpr (RPT % 8 == 0) {
#pragma unroll
    for (int i = 0; i < RPT / 8; ++i) {
      const uint4 x = __ldg(reinterpret_cast<const uint4*>(p) + i);
      w[4 * i + 0] = x.x; w[4 * i + 1] = x.y; w[4 * i + 2] = x.z; w[4 * i + 3] = x.w;
    }
  } else {
    static_assert(RPT == 4, "rows per thread: 4 or a multiple of 8");
    const uint2 x = __ldg(reinterpret_cast<const uint2*>(p));
    w[0] = x.x; w[1] = x.y;
  }
}
template <int NF>
__device__ __forceinline__ void ld_f32_rows(float (&d)[NF], const float* p) {
#pragma unroll
  for (int i = 0; i < NF / 4; ++i) {
    const float4 x = __ldg(reinterpret_cast<const float4*>(p) + i);
    d[4 * i + 0] = x.x; d[4 * i + 1] = x.y; d[4 * i + 2] = x.z; d[4 * i + 3] = x.w;
  }
}

// Inputs of one token for one thread: its RPT key rows of q, k, g, its 4 value
// columns of v (and of the gate z), and beta.
template <int RPT>
struct TokenIn {
  uint32_t q[RPT / 2], k[RPT / 2];
  float g[RPT];
  uint32_t v[2], z[2];
  float beta;
};

// ---------------------------------------------------------------- cp.async
__device__ __forceinline__ uint32_t smem_u32(const void* ptr) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(ptr));
}
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async4(uint32_t dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// ---------------------------------------------------------------- cluster
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

// ---------------------------------------------------------------- programmatic dependent launch
__device__ __forceinline__ void wait_prior_grids() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void allow_next_grid() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---------------------------------------------------------------- token staging (T > 1)
// Shared-memory image of one token's inputs for one CTA (K key rows, the
// CTA's 32 value columns).  Every member starts on a 16-byte boundary.
template <int K>
struct alignas(16) TokenSmem {
  __nv_bfloat16 q[K];
  __nv_bfloat16 k[K];
  float g[K];
  __nv_bfloat16 v[kBV];
  __nv_bfloat16 z[kBV];
  float beta[4];
};

// Issue cp.async copies of tokens [t0, t0 + cnt) into buf (all threads share the work).
template <int K, bool GATED>
__device__ __forceinline__ void stage_tokens(TokenSmem<K>* buf, const Params& p, int64_t V, int64_t n,
                                             int64_t h, int64_t col0, int64_t t0, int cnt) {
  constexpr int kQ = K * 2 / 16;    // 16-byte chunks of q (and of k)
  constexpr int kG = K * 4 / 16;    // of g
  constexpr int kV = kBV * 2 / 16;  // of v (and of z)
  constexpr int kPer = 2 * kQ + kG + 2 * kV + 1;
  for (int c = threadIdx.x; c < cnt * kPer; c += kThreads) {
    const int j = c / kPer;
    int r = c - j * kPer;
    const int64_t row = (n * p.T + t0 + j) * p.HV + h;
    TokenSmem<K>& s = buf[j];
    if (r < kQ) { cp_async16(smem_u32(s.q) + 16 * r, p.q + row * K + 8 * r); continue; }
    r -= kQ;
    if (r < kQ) { cp_async16(smem_u32(s.k) + 16 * r, p.k + row * K + 8 * r); continue; }
    r -= kQ;
    if (r < kG) { cp_async16(smem_u32(s.g) + 16 * r, p.g + row * K + 4 * r); continue; }
    r -= kG;
    if (r < kV) { cp_async16(smem_u32(s.v) + 16 * r, p.v + row * V + col0 + 8 * r); continue; }
    r -= kV;
    if (r < kV) {
      if constexpr (GATED) cp_async16(smem_u32(s.z) + 16 * r, p.gate + row * V + col0 + 8 * r);
      continue;
    }
    cp_async4(smem_u32(s.beta), p.beta + row);
  }
}

template <int RPT, int K>
__device__ __forceinline__ void read_token(TokenIn<RPT>& in, const TokenSmem<K>& s, int r0, int cq) {
  if constexpr (RPT % 8 == 0) {
#pragma unroll
    for (int i = 0; i < RPT / 8; ++i) {
      const uint4 a = *reinterpret_cast<const uint4*>(s.q + r0 + 8 * i);
      const uint4 b = *reinterpret_cast<const uint4*>(s.k + r0 + 8 * i);
      in.q[4 * i] = a.x; in.q[4 * i + 1] = a.y; in.q[4 * i + 2] = a.z; in.q[4 * i + 3] = a.w;
      in.k[4 * i] = b.x; in.k[4 * i + 1] = b.y; in.k[4 * i + 2] = b.z; in.k[4 * i + 3] = b.w;
    }
  } else {
    const uint2 a = *reinterpret_cast<const uint2*>(s.q + r0);
    const uint2 b = *reinterpret_cast<const uint2*>(s.k + r0);
    in.q[0] = a.x; in.q[1] = a.y; in.k[0] = b.x; in.k[1] = b.y;
  }
#pragma unroll
  for (int i = 0; i < RPT / 4; ++i) {
    const float4 x = *reinterpret_cast<const float4*>(s.g + r0 + 4 * i);
    in.g[4 * i] = x.x; in.g[4 * i + 1] = x.y; in.g[4 * i + 2] = x.z; in.g[4 * i + 3] = x.w;
  }
  const uint2 vv = *reinterpret_cast<const uint2*>(s.v + 4 * cq);
  const uint2 zz = *reinterpret_cast<const uint2*>(s.z + 4 * cq);
  in.v[0] = vv.x; in.v[1] = vv.y; in.z[0] = zz.x; in.z[1] = zz.y;
  in.beta = s.beta[0];
}

// ---------------------------------------------------------------- kernel
// Thread layout inside the CTA (K x 32 tile, 128 threads):
//   warp w owns key rows [w*K/4, (w+1)*K/4); inside a warp, lane = rg*8 + cq
//   with row group rg in [0,4) and column quad cq in [0,8); the thread holds
//   rows r0 .. r0+RPT-1 (r0 = w*K/4 + rg*RPT, RPT = K/16) of columns
//   4cq .. 4cq+3 of the tile.  One warp-wide float4 load covers 4 rows x 128 B.
//
// VS: the value width when fixed at compile time (row strides become
// immediates), 0 for a run-time V.  MULTI: T > 1 (tokens staged in shared
// memory); MULTI = false is the T == 1 path with all inputs in registers.
//
// Resident CTAs per SM the register budget is capped for: at K = 128 seven
// CTAs (<= 72 registers a thread) hold 1036 tiles on 148 SMs, a single wave
// for 32 sequences x 8 heads x 4 tiles.
template <int K>
struct MinBlocks {
  static constexpr int value = K >= 256 ? 3 : (K >= 128 ? 7 : 8);
};

template <int K, int VS, bool GATED, bool MULTI>
__global__ void __launch_bounds__(kThreads, (MinBlocks<K>::value))
kda_decode_kernel(const Params p) {
  constexpr int RPT = K / (kWarps * kRowGroups);
  static_assert(RPT * kWarps * kRowGroups == K && (RPT == 4 || RPT % 8 == 0), "K in {64,128,256}");

  __shared__ __align__(16) float2 red[2][kWarps][2][kColQuads * 2];  // [buf][warp][k|q][column pairs]
  __shared__ float red_qk[2][kWarps];
  __shared__ float nrm[2][kMaxClusterTiles];  // gated: per-tile sum of o^2
  __shared__ TokenSmem<K> tok[MULTI ? 2 : 1][MULTI ? kTokenChunk : 1];

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int cq = lane & (kColQuads - 1);
  const int rg = lane / kColQuads;
  const int r0 = warp * (K / kWarps) + rg * RPT;
  const int64_t V = VS ? VS : p.V;
  const int tiles = VS ? VS / kBV : p.tiles;

  const int64_t unit = blockIdx.x / tiles;  // n * HV + h
  const int tile = static_cast<int>(blockIdx.x - unit * tiles);
  const int64_t n = unit / p.HV;
  const int64_t h = unit - n * p.HV;
  const int64_t col = static_cast<int64_t>(tile) * kBV + cq * 4;
  const bool writer = (warp == 0) && (rg == 0);  // 8 lanes store the tile's 32 outputs

  wait_prior_grids();
  const int32_t slot = __ldg(p.slot_idx + n);

  // Token inputs do not depend on the slot: issue them before it lands.
  TokenIn<RPT> cur;
  if constexpr (MULTI) {
    stage_tokens<K, GATED>(tok[0], p, V, n, h, static_cast<int64_t>(tile) * kBV, 0,
                           static_cast<int>(p.T < kTokenChunk ? p.T : kTokenChunk));
    cp_async_commit();
  } else {
    const int64_t row = n * p.HV + h;  // T == 1
    ld_bf16_rows<RPT>(cur.q, p.q + row * K + r0);
    ld_bf16_rows<RPT>(cur.k, p.k + row * K + r0);
    ld_f32_rows<RPT>(cur.g, p.g + row * K + r0);
    const uint2 vv = __ldg(reinterpret_cast<const uint2*>(p.v + row * V + col));
    cur.v[0] = vv.x; cur.v[1] = vv.y;
    if constexpr (GATED) {
      const uint2 zz = __ldg(reinterpret_cast<const uint2*>(p.gate + row * V + col));
      cur.z[0] = zz.x; cur.z[1] = zz.y;
    }
    cur.beta = __ldg(p.beta + row);
  }

  if (slot < 0) {  // inactive (padding) row: zero output, pool untouched
    if constexpr (MULTI) cp_async_wait<0>();
    if (writer) {
      for (int64_t t = 0; t < p.T; ++t)
        *reinterpret_cast<uint2*>(p.out + ((n * p.T + t) * p.HV + h) * V + col) = make_uint2(0u, 0u);
    }
    return;  // uniform over the cluster: every tile of this (n, h) sees the same slot
  }

  float4* const sp =
      reinterpret_cast<float4*>(p.state + ((static_cast<int64_t>(slot) * p.HV + h) * K + r0) * V + col);
  float2 s[RPT][2];
#pragma unroll
  for (int i = 0; i < RPT; ++i) {
    const float4 x = sp[i * (V / 4)];
    s[i][0] = make_float2(x.x, x.y);
    s[i][1] = make_float2(x.z, x.w);
  }

  if constexpr (GATED) cluster_arrive_relaxed();  // peers must be running before DSMEM writes

  float2 wgt[2] = {f2(0.f), f2(0.f)};
  if constexpr (GATED) {
    const uint2 w = __ldg(reinterpret_cast<const uint2*>(p.norm_weight + col));
    wgt[0] = make_float2(bf16lo(w.x), bf16hi(w.x));
    wgt[1] = make_float2(bf16lo(w.y), bf16hi(w.y));
  }

  const float2 scale2 = f2(p.scale);
  for (int64_t t = 0; t < p.T; ++t) {
    const int buf = static_cast<int>(t & 1);
    if constexpr (MULTI) {
      const int j = static_cast<int>(t % kTokenChunk);
      const int cb = static_cast<int>((t / kTokenChunk) & 1);
      if (j == 0) {
        const int64_t next0 = t + kTokenChunk;
        if (next0 < p.T) {  // prefetch the next chunk into the other buffer
          const int64_t left = p.T - next0;
          stage_tokens<K, GATED>(tok[cb ^ 1], p, V, n, h, static_cast<int64_t>(tile) * kBV, next0,
                                 static_cast<int>(left < kTokenChunk ? left : kTokenChunk));
          cp_async_commit();
          cp_async_wait<1>();
        } else {
          cp_async_wait<0>();
        }
        __syncthreads();
      }
      read_token<RPT, K>(cur, tok[cb][j], r0, cq);
    }

    // decay and the partial reductions over this thread's rows
    float2 pk[2] = {f2(0.f), f2(0.f)}, pq[2] = {f2(0.f), f2(0.f)};
    float qk = 0.f;
#pragma unroll
    for (int i = 0; i < RPT; ++i) {
      const float qi = bf16_at(cur.q, i);
      const float ki = bf16_at(cur.k, i);
      const float2 d = f2(__expf(cur.g[i]));
      const float2 k2 = f2(ki), q2 = f2(qi);
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        s[i][j] = __fmul2_rn(s[i][j], d);
        pk[j] = __ffma2_rn(s[i][j], k2, pk[j]);
        pq[j] = __ffma2_rn(s[i][j], q2, pq[j]);
      }
      qk = fmaf(qi, ki, qk);
    }

    // Reduce-scatter across the 4 row groups of the warp: after the xor-16
    // step lanes with bit 4 clear hold S'^T k sums, set hold S'^T q; after the
    // xor-8 step each lane holds one column pair of its set.
    const bool hi16 = (lane & 16) != 0;
    const bool hi8 = (lane & 8) != 0;
    float2 keep[2], send[2];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      keep[j] = hi16 ? pq[j] : pk[j];
      send[j] = hi16 ? pk[j] : pq[j];
    }
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const float2 r = make_float2(__shfl_xor_sync(0xffffffffu, send[j].x, 16),
                                   __shfl_xor_sync(0xffffffffu, send[j].y, 16));
      keep[j] = __fadd2_rn(keep[j], r);
    }
    float2 mine = hi8 ? keep[1] : keep[0];
    const float2 other = hi8 ? keep[0] : keep[1];
    mine = __fadd2_rn(mine, make_float2(__shfl_xor_sync(0xffffffffu, other.x, 8),
                                        __shfl_xor_sync(0xffffffffu, other.y, 8)));
    qk += __shfl_xor_sync(0xffffffffu, qk, 8);
    qk += __shfl_xor_sync(0xffffffffu, qk, 16);
    red[buf][warp][hi16 ? 1 : 0][cq * 2 + (hi8 ? 1 : 0)] = mine;
    if (lane == 0) red_qk[buf][warp] = qk;
    __syncthreads();

    // across the 4 warps (fixed order: identical sums in every thread)
    float2 rk[2] = {f2(0.f), f2(0.f)}, rq[2] = {f2(0.f), f2(0.f)};
    float qkt = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      const float4 a = *reinterpret_cast<const float4*>(&red[buf][w][0][cq * 2]);
      const float4 b = *reinterpret_cast<const float4*>(&red[buf][w][1][cq * 2]);
      rk[0] = __fadd2_rn(rk[0], make_float2(a.x, a.y));
      rk[1] = __fadd2_rn(rk[1], make_float2(a.z, a.w));
      rq[0] = __fadd2_rn(rq[0], make_float2(b.x, b.y));
      rq[1] = __fadd2_rn(rq[1], make_float2(b.z, b.w));
      qkt += red_qk[buf][w];
    }

    // correction, rank-1 write, readout
    const float2 beta2 = f2(cur.beta);
    const float2 qk2 = f2(qkt);
    float2 u[2], o[2];
    const float2 vv[2] = {make_float2(bf16lo(cur.v[0]), bf16hi(cur.v[0])),
                          make_float2(bf16lo(cur.v[1]), bf16hi(cur.v[1]))};
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      u[j] = __fmul2_rn(beta2, __fadd2_rn(vv[j], make_float2(-rk[j].x, -rk[j].y)));
      o[j] = __fmul2_rn(scale2, __ffma2_rn(qk2, u[j], rq[j]));
    }
#pragma unroll
    for (int i = 0; i < RPT; ++i) {
      const float2 k2 = f2(bf16_at(cur.k, i));
#pragma unroll
      for (int j = 0; j < 2; ++j) s[i][j] = __ffma2_rn(k2, u[j], s[i][j]);
    }

    const int64_t out_row = ((n * p.T + t) * p.HV + h) * V + col;
    if constexpr (GATED) {
      // per-tile sum of o^2 (lanes 0..7 of warp 0 hold the tile's 32 outputs)
      float ss = 0.f;
      if (writer) {
        ss = o[0].x * o[0].x + o[0].y * o[0].y + o[1].x * o[1].x + o[1].y * o[1].y;
#pragma unroll
        for (int m = 1; m < kColQuads; m <<= 1) ss += __shfl_xor_sync(0x000000ffu, ss, m);
      }
      if (t == 0) cluster_wait_acquire();  // pairs with the relaxed arrive after the state loads
      if (writer && lane < tiles) {
        cluster_store_f32(cluster_map(smem_u32(&nrm[buf][tile]), static_cast<uint32_t>(lane)), ss);
      }
      cluster_arrive_release();
      cluster_wait_acquire();
      if (writer) {
        float tot = 0.f;
        for (int r = 0; r < tiles; ++r) tot += nrm[buf][r];
        const float inv = rsqrtf(tot / static_cast<float>(V) + p.eps);
        const float zz[4] = {bf16lo(cur.z[0]), bf16hi(cur.z[0]), bf16lo(cur.z[1]), bf16hi(cur.z[1])};
        const float ov[4] = {o[0].x, o[0].y, o[1].x, o[1].y};
        const float wv[4] = {wgt[0].x, wgt[0].y, wgt[1].x, wgt[1].y};
        float y[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) y[j] = ov[j] * inv * wv[j] * (1.0f / (1.0f + __expf(-zz[j])));
        *reinterpret_cast<uint2*>(p.out + out_row) = make_uint2(pack_bf16x2(y[0], y[1]), pack_bf16x2(y[2], y[3]));
      }
    } else if (writer) {
      *reinterpret_cast<uint2*>(p.out + out_row) =
          make_uint2(pack_bf16x2(o[0].x, o[0].y), pack_bf16x2(o[1].x, o[1].y));
    }
    if constexpr (!MULTI) break;  // T == 1
  }

  allow_next_grid();
#pragma unroll
  for (int i = 0; i < RPT; ++i) __stcs(sp + i * (V / 4), make_float4(s[i][0].x, s[i][0].y, s[i][1].x, s[i][1].y));
}

}  // namespace kda
