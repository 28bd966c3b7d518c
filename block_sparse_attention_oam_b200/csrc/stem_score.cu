// OAM scoring on sm_100a: the per-block pooling kernel and the block-score GEMM.
//
// Tencent Cloud article "从Stem稀疏注意力看 大模型推理的架构取舍":
//  * section "OAM：价值评估": score = routing relevance (QK^T) + beta * log||V_j||_2,
//    beta = 0.2, purely additive;
//  * section "HPC-Stem：评估选块，快几十倍": because the score is additive, compact
//    block-level representations of Q and K are computed first and one standard
//    GEMM yields every block score, with no softmax, no gather and no large
//    intermediate tensor.
// The block summary is the mean over the block's tokens; the magnitude term is the
// block mean of the per-token log L2 norm of V (zero norms clamped to FLT_MIN).
#include <cuda_fp16.h>
#include <float.h>

#include <type_traits>

#include "stem_internal.cuh"

namespace stem {
namespace {

constexpr int kPoolThreads = 128;     // at most this many threads across a token row (16 bytes each)
constexpr int kPoolCtaThreads = 512;  // threads of a pooling CTA (4 to 8 token streams)

// 16 bytes -> 8 bf16 or 16 e4m3 values as floats (FP8: the codes' values; the per-tensor
// scale is applied once per block mean or norm, not per element).
__device__ __forceinline__ void decode16(const uint4& u, float* f, bool fp8) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
  if (!fp8) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      f[2 * q] = __uint_as_float(w[q] << 16);
      f[2 * q + 1] = __uint_as_float(w[q] & 0xFFFF0000u);
    }
  } else {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
#pragma unroll
      for (int hlf = 0; hlf < 2; ++hlf) {
        uint16_t pair = static_cast<uint16_t>(w[q] >> (16 * hlf));
        uint32_t h2;
        asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(pair));
        const float2 fv = __half22float2(*reinterpret_cast<__half2*>(&h2));
        f[4 * q + 2 * hlf] = fv.x;
        f[4 * q + 2 * hlf + 1] = fv.y;
      }
    }
  }
}

// One launch pools Q (means), K (means) and V (mean log-norms): one CTA per (global block
// row, slice of one tensor's [H*d] token row); blockIdx.y runs over the Q slices, then
// K's, then V's.  A slice is up to 128 threads x 16 bytes; a narrower token row (FP8 K
// and V: 64 threads) takes fewer threads (whole warps), the CTA's 512 threads then
// covering more token streams (grp = thread / threads-per-row).  The block's tokens are
// split into contiguous runs, one per stream, each thread keeping 8 (FP8: 6) loads of 16
// bytes in flight; the streams' partial sums are added in stream order (deterministic).  A tensor
// pooled for means only adds; the V pass only forms the per-token norms.

template <int D, bool FP8>
__global__ void __launch_bounds__(kPoolCtaThreads, 2) pool_kernel(const Batch bt, const PoolSet ps) {
  constexpr int VEC = FP8 ? 16 : 8;
  constexpr int kPoolU = FP8 ? 6 : 8;  // tokens in flight per thread (FP8: 16 values each)
  constexpr int LPH = D / VEC;  // lanes per head
  constexpr int ES = FP8 ? 1 : 2;
  int ti = 0, slice = blockIdx.y;
  while (ti + 1 < ps.count && slice >= ps.t[ti].slices) slice -= ps.t[ti++].slices;
  const PoolTensor& a = ps.t[ti];
  const int HD = a.H * D;
  // threads across this slice of the token row: whole warps (32, 64, 96 or 128), so that a
  // warp never spans two token streams, whose trip counts differ on a partial block (the
  // log-norm shuffle below is warp-synchronous); lanes past the row end load nothing
  const int tpr = min(kPoolThreads, (HD / VEC + 31) / 32 * 32);
  const int streams = kPoolCtaThreads / tpr;
  const int row = blockIdx.x;
  const int b = seq_of_row(bt, row);
  const SeqInfo& s = bt.seq[b];
  const int i = row - s.row0;
  const int B = bt.block;
  const int t_beg = i * B;
  const int t_end = min(s.len, t_beg + B);
  const int n = t_end - t_beg;
  const int tx = threadIdx.x % tpr, grp = threadIdx.x / tpr;
  const int e0 = (slice * tpr + tx) * VEC;
  const bool valid = e0 < HD;
  const int h = valid ? e0 / D : 0;
  const int d0 = e0 % D;
  const unsigned char* base = static_cast<const unsigned char*>(a.x);

  float acc[VEC];
#pragma unroll
  for (int e = 0; e < VEC; ++e) acc[e] = 0.f;
  float lacc = 0.f;

  auto tok_ptr = [&](int t) -> const uint4* {
    long long rowi;
    if (a.paged) {
      // a slot outside the cache is reported (bounds error) and slot 0 read instead
      int slot = ps.block_table[static_cast<long long>(b) * ps.max_pages + t / STEM_PAGE_SIZE];
      if (slot < 0 || slot >= ps.num_slots) {
        atomicOr(ps.status, kStatusBounds);
        slot = 0;
      }
      rowi = static_cast<long long>(slot) * STEM_PAGE_SIZE + (t % STEM_PAGE_SIZE);
    } else {
      rowi = static_cast<long long>(s.tok0) + t;
    }
    return reinterpret_cast<const uint4*>(base + (rowi * HD + e0) * ES);
  };

  const int chunk = (B + streams - 1) / streams;
  const int g_beg = t_beg + grp * chunk;
  const int g_end = min(t_end, g_beg + chunk);
  // the token loop, with the per-token norms only for the tensor that needs them (V)
  auto run = [&](auto norms) {
    constexpr bool NORMS = decltype(norms)::value;
    for (int t = g_beg; t < g_end; t += kPoolU) {
      uint4 buf[kPoolU];
#pragma unroll
      for (int u = 0; u < kPoolU; ++u) {
        buf[u] = make_uint4(0, 0, 0, 0);
        if (valid && t + u < g_end) buf[u] = __ldg(tok_ptr(t + u));
      }
#pragma unroll
      for (int u = 0; u < kPoolU; ++u) {
        float f[VEC];
        decode16(buf[u], f, FP8);
        if constexpr (NORMS) {
          float ss = 0.f;
#pragma unroll
          for (int e = 0; e < VEC; ++e) ss = fmaf(f[e], f[e], ss);
#pragma unroll
          for (int o = LPH / 2; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o, LPH);
          if (t + u < g_end) lacc += logf(fmaxf(sqrtf(ss) * a.scale, FLT_MIN));
        } else {
#pragma unroll
          for (int e = 0; e < VEC; ++e) acc[e] += f[e];
        }
      }
    }
  };
  if (a.lognorm_out != nullptr)
    run(std::true_type{});
  else
    run(std::false_type{});
  // partial sums of streams 1.. to stream 0, added in stream order; [stream - 1][element]
  // [thread of the stream] (threads past the last whole stream, when tpr does not divide
  // the CTA, hold no tokens and are not added)
  __shared__ float part[(VEC + 1) * kPoolCtaThreads];
  auto slot = [&](int g, int e, int x) -> float& { return part[((g - 1) * (VEC + 1) + e) * tpr + x]; };
  if (grp > 0) {
#pragma unroll
    for (int e = 0; e < VEC; ++e) slot(grp, e, tx) = acc[e];
    slot(grp, VEC, tx) = lacc;
  }
  __syncthreads();
  if (grp > 0 || !valid) return;
  for (int g = 1; g < streams; ++g) {
#pragma unroll
    for (int e = 0; e < VEC; ++e) acc[e] += slot(g, e, tx);
    lacc += slot(g, VEC, tx);
  }
  const float inv = 1.0f / static_cast<float>(n);
  if (a.mean_out != nullptr) {
    const float mul = a.scale * inv;  // FP8: the dequantisation scale (1 for bf16)
    float* dst = a.mean_out + (static_cast<long long>(h) * bt.total_rows + row) * D + d0;
#pragma unroll
    for (int e = 0; e < VEC; e += 4)
      *reinterpret_cast<float4*>(dst + e) =
          make_float4(acc[e] * mul, acc[e + 1] * mul, acc[e + 2] * mul, acc[e + 3] * mul);
  }
  if (a.lognorm_out != nullptr && d0 == 0) a.lognorm_out[static_cast<long long>(h) * bt.total_rows + row] = lacc * inv;
}

template <int D, bool FP8>
cudaError_t pool_dispatch(const Batch& bt, PoolSet ps, cudaStream_t st) {
  constexpr int VEC = FP8 ? 16 : 8;
  int slices = 0;
  for (int t = 0; t < ps.count; ++t) {
    const int hd = ps.t[t].H * D;
    // a tensor is pooled for its means or for its norms, not both
    if ((ps.t[t].mean_out == nullptr) == (ps.t[t].lognorm_out == nullptr)) return cudaErrorInvalidValue;
    ps.t[t].slices = (hd + kPoolThreads * VEC - 1) / (kPoolThreads * VEC);
    slices += ps.t[t].slices;
  }
  dim3 grid(bt.total_rows, slices);
  pool_kernel<D, FP8><<<grid, kPoolCtaThreads, 0, st>>>(bt, ps);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ scores
// One CTA per (64 x 64 lower-triangular tile of one sequence, q-head), each thread a 4 x 4
// block of consecutive rows and columns.  fp32 SIMT:
// the GEMM is N x N x d per head (about 4 GFLOP at 128K), far below the path's
// cost, and fp32 keeps the scores within 1e-3 relative of the float64 definition.
constexpr int kTile = 64;
constexpr int kKc = 32;

__global__ void __launch_bounds__(256) score_kernel(const Batch bt, const float* __restrict__ qbar,
                                                    const float* __restrict__ kbar,
                                                    const float* __restrict__ lbar, int Hq, int Hkv, int D,
                                                    float sigma, float beta, float* __restrict__ scores) {
  // [d][row] with rows padded to 68 floats: a thread's 4 consecutive rows (or columns) are
  // one 16-byte read
  __shared__ __align__(16) float Qs[kKc][kTile + 4];
  __shared__ __align__(16) float Ks[kKc][kTile + 4];
  const int h = blockIdx.y;
  const int kh = h / (Hq / Hkv);
  // decode (sequence, tile row, tile col)
  long long t = blockIdx.x;
  int b = 0;
  int nt = 0;
  for (; b < bt.num_seqs; ++b) {
    nt = (bt.seq[b].nblk + kTile - 1) / kTile;
    long long cnt = static_cast<long long>(nt) * (nt + 1) / 2;
    if (t < cnt) break;
    t -= cnt;
  }
  if (b >= bt.num_seqs) return;
  int ti = static_cast<int>((sqrt(8.0 * static_cast<double>(t) + 1.0) - 1.0) * 0.5);
  while (static_cast<long long>(ti) * (ti + 1) / 2 > t) --ti;
  while (static_cast<long long>(ti + 1) * (ti + 2) / 2 <= t) ++ti;
  const int tj = static_cast<int>(t - static_cast<long long>(ti) * (ti + 1) / 2);
  const SeqInfo& s = bt.seq[b];
  const int N = s.nblk;
  const int R = bt.total_rows;
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  const int i0 = ti * kTile, j0 = tj * kTile;

  float acc[4][4];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int c = 0; c < 4; ++c) acc[a][c] = 0.f;

  const float* qrow = qbar + (static_cast<long long>(h) * R + s.row0) * D;
  const float* krow = kbar + (static_cast<long long>(kh) * R + s.row0) * D;
  const int lr = threadIdx.x / 4;        // 0..63 tile row loaded by this thread
  const int lc = (threadIdx.x % 4) * 8;  // 8 consecutive d of the chunk
  for (int kc = 0; kc < D; kc += kKc) {
    float4 qa = make_float4(0, 0, 0, 0), qb = qa, ka = qa, kb = qa;
    if (i0 + lr < N) {
      const float4* p = reinterpret_cast<const float4*>(qrow + static_cast<long long>(i0 + lr) * D + kc + lc);
      qa = p[0];
      qb = p[1];
    }
    if (j0 + lr < N) {
      const float4* p = reinterpret_cast<const float4*>(krow + static_cast<long long>(j0 + lr) * D + kc + lc);
      ka = p[0];
      kb = p[1];
    }
    __syncthreads();
    const float qv[8] = {qa.x, qa.y, qa.z, qa.w, qb.x, qb.y, qb.z, qb.w};
    const float kv[8] = {ka.x, ka.y, ka.z, ka.w, kb.x, kb.y, kb.z, kb.w};
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      Qs[lc + e][lr] = qv[e];
      Ks[lc + e][lr] = kv[e];
    }
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < kKc; ++kk) {
      const float4 a4 = *reinterpret_cast<const float4*>(&Qs[kk][4 * ty]);
      const float4 b4 = *reinterpret_cast<const float4*>(&Ks[kk][4 * tx]);
      const float av[4] = {a4.x, a4.y, a4.z, a4.w}, bv[4] = {b4.x, b4.y, b4.z, b4.w};
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[a][c] = fmaf(av[a], bv[c], acc[a][c]);
    }
  }
  float* out = scores + static_cast<long long>(h) * bt.scores_per_head + s.score0;
  const float* lb = lbar + static_cast<long long>(kh) * R + s.row0;
#pragma unroll
  for (int a = 0; a < 4; ++a) {
    const int i = i0 + 4 * ty + a;
    if (i >= N) continue;
    const long long roff = static_cast<long long>(i) * (i + 1) / 2;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int j = j0 + 4 * tx + c;
      if (j <= i) out[roff + j] = fmaf(sigma, acc[a][c], beta * lb[j]);
    }
  }
}

}  // namespace

cudaError_t launch_pool(const Batch& bt, const PoolSet& ps, int head_dim, bool fp8, cudaStream_t st) {
  if (ps.count < 1 || ps.count > 3) return cudaErrorInvalidValue;
  if (head_dim == 128) return fp8 ? pool_dispatch<128, true>(bt, ps, st) : pool_dispatch<128, false>(bt, ps, st);
  if (head_dim == 64 && !fp8) return pool_dispatch<64, false>(bt, ps, st);
  return cudaErrorInvalidValue;
}

cudaError_t launch_score(const Batch& bt, const float* qbar, const float* kbar, const float* lbar, int Hq, int Hkv,
                         int head_dim, float sigma, float beta, float* scores, cudaStream_t st) {
  long long tiles = 0;
  for (int b = 0; b < bt.num_seqs; ++b) {
    long long nt = (bt.seq[b].nblk + kTile - 1) / kTile;
    tiles += nt * (nt + 1) / 2;
  }
  dim3 grid(static_cast<unsigned>(tiles), Hq);
  score_kernel<<<grid, 256, 0, st>>>(bt, qbar, kbar, lbar, Hq, Hkv, head_dim, sigma, beta, scores);
  return cudaGetLastError();
}

}  // namespace stem
