// TPD budget generation fused with the per-row top-k (sm_100a).
//
// Tencent Cloud article "从Stem稀疏注意力看 大模型推理的架构取舍":
//  * section "TPD：优先级排序": the top-k budget decays linearly from the initial
//    position to the end (the end keeps mu = 0.7 of the initial budget) and the
//    total is only redistributed;
//  * section "HPC-Stem：评估选块，快几十倍": budget generation and the selection sort
//    are fused into one operator so the budget never round-trips through HBM;
//  * section "用架构师的眼睛看稀疏注意力": the initial tokens are the trunk every
//    output depends on, so block 0 is always kept (and so is the diagonal block).
//
// One CTA per (global block row, group of 8 lists).  The CTA recomputes the row's
// budget k_i and its CSR offset sum_{i'<i} k_i' from r_start (fp64, the same
// operation order as the host planner), then each warp selects one list's row (a
// list per q-head, or — shared lists, an extension of this library — a list per KV
// group ranked by the float32 sum, in head order, of its q-heads' scores):
// a most-significant-digit-first radix select (4 passes of 8 bits, histogram in
// shared memory) finds the k-th largest order-preserving score key, and a
// ballot-based compaction walks the candidates in ascending block order, taking
// every key above the threshold and the lowest-index keys equal to it.
#include "stem_internal.cuh"

namespace stem {
namespace {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;

// Order-preserving map float -> uint32 (larger score -> larger key).  NaN ranks as
// -inf and -0 as +0, so the ranking equals (score descending, index ascending).
__device__ __forceinline__ uint32_t score_key(float f) {
  uint32_t bits = __float_as_uint(f);
  if ((bits & 0x7FFFFFFFu) > 0x7F800000u) bits = 0xFF800000u;
  if (bits == 0x80000000u) bits = 0u;
  return (bits & 0x80000000u) ? ~bits : (bits | 0x80000000u);
}

// Budget and CSR offset of one block row, computed by all NT threads of the CTA (fp64,
// the host planner's operation order).  Writes row_ptr for the row (and the final entry)
// when `write` is set.  *ok is false (and the status word flagged) if the row's list
// would overrun its sequence's share of col_idx.
struct RowPlan {
  int b, i, N, k_i;
  long long off;   // offset of the row's list inside its sequence's lists
};

template <int NT>
__device__ __forceinline__ RowPlan plan_row(const Batch& bt, int row, bool write, int32_t* row_ptr, uint32_t* status,
                                            long long* red, bool* ok) {
  const int b = seq_of_row(bt, row);
  const SeqInfo& s = bt.seq[b];
  const int i = row - s.row0;
  const int N = s.nblk;
  const int k_i = tpd_k(s.r_start, N, bt.mu, i);
  long long part = 0;
  for (int ii = threadIdx.x; ii < i; ii += NT) part += tpd_k(s.r_start, N, bt.mu, ii);
  for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  if (lane == 0) red[warp] = part;
  __syncthreads();
  long long off = 0;
  for (int w = 0; w < NT / 32; ++w) off += red[w];
  *ok = off + k_i <= s.nnz;
  if (!*ok) {
    if (threadIdx.x == 0) atomicOr(status, kStatusBounds);
  } else if (write && threadIdx.x == 0) {
    row_ptr[row] = static_cast<int32_t>(s.nnz0 + off);
    if (b == bt.num_seqs - 1 && i == N - 1) row_ptr[row + 1] = static_cast<int32_t>(s.nnz0 + off + k_i);
  }
  return RowPlan{b, i, N, k_i, off};
}

// Lists that need no ranking: row 0, budgets of the forced blocks only, and rows that
// keep every block.  One warp writes the list; returns true when it did.
__device__ __forceinline__ bool trivial_list(int i, int k_i, int32_t* out, int lane) {
  if (i == 0) {
    if (lane == 0) out[0] = 0;
    return true;
  }
  const int need = k_i - 2;  // blocks to choose among 1..i-1
  if (need <= 0) {
    if (lane == 0) {
      out[0] = 0;
      out[1] = i;
    }
    return true;
  }
  if (need >= i - 1) {
    for (int j = lane; j <= i; j += 32) out[j] = j;
    return true;
  }
  return false;
}

// One warp ranks keys[1..i-1] (order-preserving score keys) and writes the list: block 0,
// the `need` best candidates under (key descending, index ascending), block i.  A
// most-significant-digit-first radix select (8-bit digits below the bits all candidates
// share, histogram in shared memory) finds the need-th largest key, then a ballot compaction walks the candidates in
// ascending block order, taking every key above it and the lowest-index keys equal to it.
// (Measured slower for the 128K layer: a one-bit-at-a-time select with warp-reduced
// counts and no atomics, 0.22 ms, and one atomic per distinct digit of a warp's keys
// (match.any), 0.19 ms, against 0.14 ms.)
__device__ __forceinline__ void select_warp(const uint32_t* keys, uint32_t* hist, int i, int need, int32_t* out,
                                            int lane) {
  const unsigned full = 0xffffffffu;
  // the bits every candidate key shares are fixed at once (a row's scores share their
  // sign and leading exponent bits); the 8-bit digits start below them, so the first pass
  // spreads the keys over many bins instead of piling them into one or two
  uint32_t kmin = 0xFFFFFFFFu, kmax = 0u;
  for (int j = 1 + lane; j < i; j += 32) {
    const uint32_t u = keys[j];
    kmin = min(kmin, u);
    kmax = max(kmax, u);
  }
  kmin = __reduce_min_sync(full, kmin);
  kmax = __reduce_max_sync(full, kmax);
  const uint32_t diff = kmin ^ kmax;
  const int top = diff != 0u ? 31 - __clz(diff) : -1;            // highest bit the keys differ in
  uint32_t pmask = top >= 0 ? ~((2u << top) - 1u) : 0xFFFFFFFFu;  // 2u << 31 wraps to 0: no common bits
  uint32_t prefix = kmin & pmask;
  int rem = need;
  for (int hi = top; hi >= 0; hi -= 8) {
    const int shift = hi >= 7 ? hi - 7 : 0;
    const uint32_t dmask = (2u << (hi - shift)) - 1u;              // digit of hi - shift + 1 <= 8 bits
    for (int q = lane; q < 256; q += 32) hist[q] = 0;
    __syncwarp();
    for (int j = 1 + lane; j < i; j += 32) {
      const uint32_t u = keys[j];
      if ((u & pmask) == prefix) atomicAdd(&hist[(u >> shift) & dmask], 1u);
    }
    __syncwarp();
    int c[8];
    int tot = 0;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      c[q] = static_cast<int>(hist[8 * lane + q]);
      tot += c[q];
    }
    // inclusive suffix sum over lanes lane..31
    int incl = tot;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_down_sync(full, incl, o);
      if (lane + o < 32) incl += y;
    }
    int above = incl - tot;  // keys in digits owned by higher lanes
    int found = -1, found_above = 0;
#pragma unroll
    for (int q = 7; q >= 0; --q) {
      if (found < 0 && above < rem && rem <= above + c[q]) {
        found = 8 * lane + q;
        found_above = above;
      }
      above += c[q];
    }
    const unsigned bal = __ballot_sync(full, found >= 0);
    const int src = __ffs(bal) - 1;
    const int digit = __shfl_sync(full, found, src);
    rem -= __shfl_sync(full, found_above, src);
    prefix |= static_cast<uint32_t>(digit) << shift;
    pmask |= dmask << shift;
    __syncwarp();
  }
  // prefix = key of the need-th best candidate; rem = how many keys equal to it to take
  const unsigned lt = (1u << lane) - 1u;
  int pos = 1, eq_seen = 0;
  if (lane == 0) out[0] = 0;
  for (int base = 1; base < i; base += 32) {
    const int j = base + lane;
    const bool in = j < i;
    const uint32_t u = in ? keys[j] : 0u;
    const bool gt = in && u > prefix;
    const bool eq = in && u == prefix;
    const unsigned eqb = __ballot_sync(full, eq);
    const bool take = gt || (eq && eq_seen + __popc(eqb & lt) < rem);
    const unsigned tb = __ballot_sync(full, take);
    if (take) out[pos + __popc(tb & lt)] = j;
    pos += __popc(tb);
    eq_seen += __popc(eqb);
  }
  if (lane == 0) out[pos] = i;
}

__global__ void __launch_bounds__(kThreads) select_kernel(const Batch bt, const float* __restrict__ scores,
                                                          int Hq, int group, int32_t* __restrict__ row_ptr,
                                                          int32_t* __restrict__ col_idx, uint32_t* status) {
  extern __shared__ uint32_t sm[];
  uint32_t* hist_all = sm;                              // [kWarps][256]
  uint32_t* keys_all = sm + kWarps * 256;               // [kWarps][STEM_MAX_BLOCKS]
  __shared__ long long red[kWarps];

  const int row = blockIdx.x;
  bool ok;
  const RowPlan rp = plan_row<kThreads>(bt, row, blockIdx.y == 0, row_ptr, status, red, &ok);
  if (!ok) return;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int h = blockIdx.y * kWarps + warp;  // list index
  if (h >= Hq / group) return;
  const SeqInfo& s = bt.seq[rp.b];
  const int i = rp.i;
  int32_t* out = col_idx + static_cast<long long>(h) * bt.nnz_per_head + s.nnz0 + rp.off;
  if (trivial_list(i, rp.k_i, out, lane)) return;

  const float* srow = scores + static_cast<long long>(h) * group * bt.scores_per_head + s.score0 +
                      static_cast<long long>(i) * (i + 1) / 2;
  uint32_t* keys = keys_all + warp * STEM_MAX_BLOCKS;
  uint32_t* hist = hist_all + warp * 256;
  for (int j = 1 + lane; j < i; j += 32) {
    float v = srow[j];
    for (int t = 1; t < group; ++t) v = __fadd_rn(v, srow[static_cast<long long>(t) * bt.scores_per_head + j]);
    keys[j] = score_key(v);
  }
  __syncwarp();
  select_warp(keys, hist, i, rp.k_i - 2, out, lane);
}

// ------------------------------------------------------- fused score + select
// Tencent Cloud article "从Stem稀疏注意力看 大模型推理的架构取舍", section
// "HPC-Stem：评估选块，快几十倍": the block scores come straight from the compact
// block summaries and feed the budgeted top-k in the same operator, with no score
// matrix in between.  One CTA per (block row, kv-head, group of up to 4 lists): it
// stages the kv-head's block means K̄ in shared memory 128 blocks at a time, each thread
// scores one candidate block for every q-head the CTA needs,
//   s = fmaf(sigma, <Q̄_i, K̄_j>, beta * l̄_j),  the dot product a float32 fma chain over
// d in index order (the same operations, in the same order, as score_kernel, so the
// keys equal those of the score matrix bit for bit), and one warp per list ranks them.
constexpr int kFusedThreads = 128;
constexpr int kFusedChunk = 128;      // candidate blocks staged per round (one per thread)
constexpr int kFusedMaxHeads = 16;    // q-heads whose Q̄ rows a CTA holds (shared lists: the group)

template <int D>
struct FusedSmem {
  static constexpr int KS = D + 4;    // padded K̄ row (floats): conflict-free 16-byte reads
  static constexpr size_t K_OFF = 0;
  static constexpr size_t Q_OFF = K_OFF + sizeof(float) * kFusedChunk * KS;
  static constexpr size_t KEY_OFF = Q_OFF + sizeof(float) * kFusedMaxHeads * D;
  static constexpr size_t HIST_OFF = KEY_OFF + sizeof(uint32_t) * 4 * STEM_MAX_BLOCKS;
  static constexpr size_t BYTES = HIST_OFF + sizeof(uint32_t) * 4 * 256;
};

template <int D>
__global__ void __launch_bounds__(kFusedThreads) select_fused_kernel(
    const Batch bt, const float* __restrict__ qbar, const float* __restrict__ kbar, const float* __restrict__ lbar,
    int Hq, int Hkv, int group, float sigma, float beta, int32_t* __restrict__ row_ptr,
    int32_t* __restrict__ col_idx, uint32_t* status) {
  using L = FusedSmem<D>;
  extern __shared__ __align__(16) unsigned char fsm[];
  float* Ks = reinterpret_cast<float*>(fsm + L::K_OFF);
  float* Qs = reinterpret_cast<float*>(fsm + L::Q_OFF);
  uint32_t* keys_all = reinterpret_cast<uint32_t*>(fsm + L::KEY_OFF);
  uint32_t* hist_all = reinterpret_cast<uint32_t*>(fsm + L::HIST_OFF);
  __shared__ long long red[kFusedThreads / 32];

  const int row = blockIdx.x, kh = blockIdx.y, z = blockIdx.z;
  bool ok;
  const RowPlan rp = plan_row<kFusedThreads>(bt, row, kh == 0 && z == 0, row_ptr, status, red, &ok);
  if (!ok) return;
  const int g = Hq / Hkv;
  const bool shared_lists = group > 1;
  // lists of this CTA and the q-heads they rank
  const int nlists = shared_lists ? 1 : min(4, g - 4 * z);
  const int h0 = kh * g + (shared_lists ? 0 : 4 * z);   // first q-head scored
  const int nheads = shared_lists ? g : nlists;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const SeqInfo& s = bt.seq[rp.b];
  const int i = rp.i;
  const int list0 = shared_lists ? kh : h0;
  auto list_out = [&](int w) {
    return col_idx + static_cast<long long>(list0 + w) * bt.nnz_per_head + s.nnz0 + rp.off;
  };
  // rows that need no ranking (the same for every list of the row)
  if (i == 0 || rp.k_i - 2 <= 0 || rp.k_i - 2 >= i - 1) {
    if (warp < nlists) trivial_list(i, rp.k_i, list_out(warp), lane);
    return;
  }
  const int R = bt.total_rows;
  const long long grow = s.row0 + i;
  // the Q̄ rows of the scored heads
  for (int e = threadIdx.x; e < nheads * D; e += kFusedThreads) {
    const int hh = e / D, d = e % D;
    Qs[e] = qbar[(static_cast<long long>(h0 + hh) * R + grow) * D + d];
  }
  const float* kb = kbar + (static_cast<long long>(kh) * R + s.row0) * D;
  const float* lb = lbar + static_cast<long long>(kh) * R + s.row0;
  for (int j0 = 1; j0 < i; j0 += kFusedChunk) {
    const int nj = min(kFusedChunk, i - j0);
    __syncthreads();  // the previous chunk's K̄ rows are no longer read
    for (int e = threadIdx.x; e < nj * (D / 4); e += kFusedThreads) {
      const int r = e / (D / 4), c = e % (D / 4);
      *reinterpret_cast<float4*>(Ks + r * L::KS + 4 * c) =
          *reinterpret_cast<const float4*>(kb + static_cast<long long>(j0 + r) * D + 4 * c);
    }
    __syncthreads();
    const int jr = threadIdx.x;
    if (jr < nj) {
      const int j = j0 + jr;
      const float* krow = Ks + jr * L::KS;
      const float bl = beta * lb[j];
      float v = 0.f;  // shared lists: the group's float32 sum in head order
      for (int hb = 0; hb < nheads; hb += 4) {
        // four heads at a time (missing ones read a valid row and are discarded)
        const float* q0 = Qs + min(hb, nheads - 1) * D;
        const float* q1 = Qs + min(hb + 1, nheads - 1) * D;
        const float* q2 = Qs + min(hb + 2, nheads - 1) * D;
        const float* q3 = Qs + min(hb + 3, nheads - 1) * D;
        float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll 8
        for (int d = 0; d < D; d += 4) {
          const float4 k4 = *reinterpret_cast<const float4*>(krow + d);
          const float4 x0 = *reinterpret_cast<const float4*>(q0 + d);
          const float4 x1 = *reinterpret_cast<const float4*>(q1 + d);
          const float4 x2 = *reinterpret_cast<const float4*>(q2 + d);
          const float4 x3 = *reinterpret_cast<const float4*>(q3 + d);
          a0 = fmaf(x0.x, k4.x, a0); a0 = fmaf(x0.y, k4.y, a0); a0 = fmaf(x0.z, k4.z, a0); a0 = fmaf(x0.w, k4.w, a0);
          a1 = fmaf(x1.x, k4.x, a1); a1 = fmaf(x1.y, k4.y, a1); a1 = fmaf(x1.z, k4.z, a1); a1 = fmaf(x1.w, k4.w, a1);
          a2 = fmaf(x2.x, k4.x, a2); a2 = fmaf(x2.y, k4.y, a2); a2 = fmaf(x2.z, k4.z, a2); a2 = fmaf(x2.w, k4.w, a2);
          a3 = fmaf(x3.x, k4.x, a3); a3 = fmaf(x3.y, k4.y, a3); a3 = fmaf(x3.z, k4.z, a3); a3 = fmaf(x3.w, k4.w, a3);
        }
        const float acc[4] = {a0, a1, a2, a3};
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          if (hb + u < nheads) {
            const float sc = fmaf(sigma, acc[u], bl);
            if (shared_lists) {
              v = hb + u == 0 ? sc : __fadd_rn(v, sc);
            } else {
              keys_all[u * STEM_MAX_BLOCKS + j] = score_key(sc);
            }
          }
        }
      }
      if (shared_lists) keys_all[j] = score_key(v);
    }
  }
  __syncthreads();
  if (warp < nlists)
    select_warp(keys_all + warp * STEM_MAX_BLOCKS, hist_all + warp * 256, i, rp.k_i - 2, list_out(warp), lane);
}

template <int D>
cudaError_t launch_fused(const Batch& bt, const float* qbar, const float* kbar, const float* lbar, int Hq, int Hkv,
                         int group, float sigma, float beta, int32_t* row_ptr, int32_t* col_idx, uint32_t* status,
                         cudaStream_t st) {
  const size_t smem = FusedSmem<D>::BYTES;
  cudaError_t e = set_smem_once<select_fused_kernel<D>>(static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int g = Hq / Hkv;
  dim3 grid(bt.total_rows, Hkv, group > 1 ? 1 : (g + 3) / 4);
  select_fused_kernel<D><<<grid, kFusedThreads, smem, st>>>(bt, qbar, kbar, lbar, Hq, Hkv, group, sigma, beta,
                                                            row_ptr, col_idx, status);
  return cudaGetLastError();
}

}  // namespace

bool fused_select_supported(int Hq, int Hkv, int group, int head_dim) {
  return (head_dim == 64 || head_dim == 128) && (group == 1 || Hq / Hkv <= kFusedMaxHeads);
}

cudaError_t launch_select_fused(const Batch& bt, const float* qbar, const float* kbar, const float* lbar, int Hq,
                                int Hkv, int group, int head_dim, float sigma, float beta, int32_t* row_ptr,
                                int32_t* col_idx, uint32_t* status, cudaStream_t st) {
  if (!fused_select_supported(Hq, Hkv, group, head_dim)) return cudaErrorInvalidValue;
  if (head_dim == 128)
    return launch_fused<128>(bt, qbar, kbar, lbar, Hq, Hkv, group, sigma, beta, row_ptr, col_idx, status, st);
  return launch_fused<64>(bt, qbar, kbar, lbar, Hq, Hkv, group, sigma, beta, row_ptr, col_idx, status, st);
}

cudaError_t launch_select(const Batch& bt, const float* scores, int Hq, int group, int32_t* row_ptr,
                          int32_t* col_idx, uint32_t* status, cudaStream_t st) {
  const size_t smem = static_cast<size_t>(kWarps) * (256 + STEM_MAX_BLOCKS) * sizeof(uint32_t);
  cudaError_t e = set_smem_once<select_kernel>(static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  dim3 grid(bt.total_rows, (Hq / group + kWarps - 1) / kWarps);
  select_kernel<<<grid, kThreads, smem, st>>>(bt, scores, Hq, group, row_ptr, col_idx, status);
  return cudaGetLastError();
}

}  // namespace stem
