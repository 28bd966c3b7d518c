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

__global__ void __launch_bounds__(kThreads) select_kernel(const Batch bt, const float* __restrict__ scores,
                                                          int Hq, int group, int32_t* __restrict__ row_ptr,
                                                          int32_t* __restrict__ col_idx, uint32_t* status) {
  extern __shared__ uint32_t sm[];
  uint32_t* hist_all = sm;                              // [kWarps][256]
  uint32_t* keys_all = sm + kWarps * 256;               // [kWarps][STEM_MAX_BLOCKS]
  __shared__ long long red[kWarps];

  const int row = blockIdx.x;
  const int b = seq_of_row(bt, row);
  const SeqInfo& s = bt.seq[b];
  const int i = row - s.row0;
  const int N = s.nblk;
  const int k_i = tpd_k(s.r_start, N, bt.mu, i);

  // CSR offset of this row inside the sequence: sum of the budgets of rows < i.
  long long part = 0;
  for (int ii = threadIdx.x; ii < i; ii += kThreads) part += tpd_k(s.r_start, N, bt.mu, ii);
  for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  if (lane == 0) red[warp] = part;
  __syncthreads();
  long long off = 0;
  for (int w = 0; w < kWarps; ++w) off += red[w];

  const bool ok = off + k_i <= s.nnz;
  if (!ok) {
    if (threadIdx.x == 0) atomicOr(status, kStatusBounds);
    return;
  }
  if (blockIdx.y == 0 && threadIdx.x == 0) {
    row_ptr[row] = static_cast<int32_t>(s.nnz0 + off);
    if (b == bt.num_seqs - 1 && i == N - 1) row_ptr[row + 1] = static_cast<int32_t>(s.nnz0 + off + k_i);
  }

  const int h = blockIdx.y * kWarps + warp;  // list index
  if (h >= Hq / group) return;
  int32_t* out = col_idx + static_cast<long long>(h) * bt.nnz_per_head + s.nnz0 + off;
  const unsigned full = 0xffffffffu;
  if (i == 0) {
    if (lane == 0) out[0] = 0;
    return;
  }
  const int forced = 2;
  const int need = k_i - forced;  // blocks to choose among 1..i-1
  if (need <= 0) {
    if (lane == 0) {
      out[0] = 0;
      out[1] = i;
    }
    return;
  }
  if (need >= i - 1) {  // every block of the row
    for (int j = lane; j <= i; j += 32) out[j] = j;
    return;
  }

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

  uint32_t prefix = 0, pmask = 0;
  int rem = need;
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int q = lane; q < 256; q += 32) hist[q] = 0;
    __syncwarp();
    for (int j = 1 + lane; j < i; j += 32) {
      const uint32_t u = keys[j];
      if ((u & pmask) == prefix) atomicAdd(&hist[(u >> shift) & 255u], 1u);
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
    pmask |= 0xFFu << shift;
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

}  // namespace

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
