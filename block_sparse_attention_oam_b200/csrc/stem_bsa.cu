// Block-sparse causal flash-attention prefill on sm_100a (tcgen05 + TMEM + TMA).
//
// Tencent Cloud article "从Stem稀疏注意力看 大模型推理的架构取舍", section
// "HPC-BSA：跳块零开销的秘密": for each Q block the kernel holds the list of KV
// blocks to visit and its inner loop walks only that list, with no per-block
// "skip?" branch; a skipped block is mathematically the same as all its scores
// being -inf, so the softmax stays exact; the inner path is the dense one.  The
// same section notes native support for a paged KV cache.
//
// Design (one CTA per SM, persistent over (q-head, q-block) tiles, 10 warps):
//   warp 0      TMA producer: the Q tile once per tile, then K_j and V_j of every listed
//               block into separate rings (64-row boxes, 128-byte swizzle; a paged cache
//               is read page by page through the block table).
//   warp 1      MMA issuer (one thread): S = Q K_j^T into one of two TMEM S buffers, then
//               O += P_j V_j with P read from TMEM (where the softmax wrote it over S_j)
//               and V from shared memory.  S_{j+1} is issued before P_j is ready, so the
//               tensor core overlaps the softmax.
//   warps 2..9  softmax, two warpgroups: each query row is shared by two threads, one per
//               warpgroup, each owning half of every KV block's columns.  The halves run
//               independent online softmaxes (own running max, own sum, own O accumulator
//               in TMEM) and are merged once per tile in the epilogue, so no per-block
//               exchange between them is needed.  Log2 domain, packed fp32x2 arithmetic;
//               the token-level causal mask only on the diagonal block (always the last
//               list entry); lazy rescaling of O (only when a running max grows by more
//               than 2^8), waiting for the previous P V product only then; O normalised
//               by the sum of the rounded P weights the product used.
// Every wait is bounded (2 s); on expiry the CTA raises an abort flag, records
// STEM_ERR_TIMEOUT in the status word, drains its tensor-core work, waits (bounded)
// for its copies and releases its TMEM before exiting.
#include <string.h>

#include <type_traits>

#include "stem_internal.cuh"

namespace stem {
namespace {

constexpr int kBM = 128;              // query rows per tile (tcgen05 M)
constexpr int kSoftmaxWarps = 8;
constexpr int kThreads = 64 + 32 * kSoftmaxWarps;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kSmemCap = 227 * 1024;

template <int D, int BN, bool FP8>
struct Cfg {
  static constexpr int ES = FP8 ? 1 : 2;
  static constexpr int CH = 128 / ES;             // elements per 128-byte swizzle row
  static constexpr int DCH = D * ES / 128;        // 128-byte chunks along d
  static_assert(D * ES % 128 == 0 && BN * ES % 128 == 0, "rows must be whole 128-byte swizzle rows");
  static constexpr int Q_CHUNK = kBM * 128;
  static constexpr int KV_CHUNK = BN * 128;
  static constexpr int Q_BYTES = kBM * D * ES;
  static constexpr int KV_BYTES = BN * D * ES;
  static constexpr int S_KSTEPS = D * ES / 32;    // MMAs along d for S (32 bytes of K each)
  static constexpr int PV_KSTEPS = BN * ES / 32;  // MMAs along the KV block for O
  static constexpr int PV_KROWS = 32 / ES;        // KV rows consumed per PV MMA
  static constexpr int HALVES = BN / 64;          // 64-row TMA boxes per KV block
  static constexpr int HALF = BN / 2;             // S columns per softmax thread
  static constexpr int P_COLS = HALF * ES / 4;    // TMEM columns of one thread's P (packed)
  static constexpr int O_HALF = D / 2;            // output columns stored per softmax thread
  static constexpr int PV_HSTEPS = PV_KSTEPS / 2; // P V MMAs per half (one O accumulator each)
  static constexpr int EXTRA = 512 + 3072;        // barriers, per-tile (m, l, lt) exchange
  static constexpr int SLACK = 1024;              // alignment of the tiles to 1024 bytes
  // K / V ring depths: as deep as shared memory allows, at most 4
  static constexpr int ROOM = static_cast<int>(kSmemCap) - Q_BYTES - EXTRA - SLACK;
  static constexpr int KST = ROOM / KV_BYTES >= 8 ? 4 : (ROOM / KV_BYTES >= 6 ? 3 : 2);
  static constexpr int VST = ROOM / KV_BYTES >= 8 ? 4 : (ROOM / KV_BYTES >= 5 ? (ROOM / KV_BYTES) - KST : 2);
  static_assert(KST + VST <= ROOM / KV_BYTES, "K/V rings do not fit");
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + Q_BYTES;
  static constexpr int OFF_V = OFF_K + KST * KV_BYTES;
  static constexpr int OFF_BAR = OFF_V + VST * KV_BYTES;
  static constexpr int OFF_XCH = OFF_BAR + 512;    // float [3 kind][2 wg][128]
  static constexpr int SMEM = OFF_XCH + 3072 + SLACK;
  // force one CTA per SM (the TMEM allocation takes all 512 columns)
  static constexpr int SMEM_LAUNCH = SMEM < 120 * 1024 ? 120 * 1024 : SMEM;
  static_assert(SMEM <= static_cast<int>(kSmemCap), "shared memory budget exceeded");
  static constexpr uint32_t FMT = FP8 ? 0u : 1u;  // e4m3 (kind::f8f6f4) or bf16 (kind::f16)
  static constexpr uint32_t IDESC_S = instr_desc(FMT, 0, 0, kBM, BN);
  static constexpr uint32_t IDESC_PV = instr_desc(FMT, 0, 1, kBM, D);
};

struct BsaParams {
  CUtensorMap tq;   // Q  [T, Hq, d]: dims (d, Hq, T), box (CH, 1, 128)
  CUtensorMap tk;   // K  [rows, Hkv, d]: dims (d, Hkv, rows), box (CH, 1, 64)
  CUtensorMap tv;   // V  same as K
  Batch bt;
  const int32_t* row_ptr;
  const int32_t* col_idx;
  const int32_t* block_table;
  int max_pages;
  int num_slots;
  void* out;
  float* lse;
  int Hq, Hkv;
  int total_tiles;
  float scale_log2;  // sigma * q_scale * k_scale * log2(e)
  float p_bias;      // log2 of the factor P is scaled by before rounding (FP8: log2 1.75)
  float out_scale;   // FP8: v_scale (l carries the P factor); BF16: 1
  float p_scale;     // the factor itself (1 for BF16)
  uint32_t* status;
  int inject;        // 1: CTA 0 withholds its first K tile (failure-detection test)
  signed char order[STEM_MAX_SEQS];  // sequences by decreasing block count
};

struct Tile {
  int b, i, h;
};

// Tile order: sequences by decreasing length; inside a sequence kv-head by kv-head, rows
// from the last (longest list) to the first, the g q-heads of a row adjacent.  The CTAs
// running at one time then share one kv-head's K/V, which fits in L2.
__device__ __forceinline__ Tile decode_tile(const BsaParams& p, int t) {
  Tile r{0, 0, 0};
  const int G = p.Hq / p.Hkv;
  int acc = 0;
  for (int q = 0; q < p.bt.num_seqs; ++q) {
    const int b = p.order[q];
    const int nb = p.bt.seq[b].nblk;
    const int nt = nb * p.Hq;
    if (t < acc + nt) {
      const int local = t - acc;
      const int kvh = local / (nb * G);
      const int rem = local - kvh * nb * G;
      r.b = b;
      r.i = nb - 1 - rem / G;
      r.h = kvh * G + rem % G;
      return r;
    }
    acc += nt;
  }
  return r;
}

// Warp-uniform bounded wait on an mbarrier phase.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          uint32_t* status) {
  const unsigned full = 0xffffffffu;
  if (__all_sync(full, mbar_try_wait(bar, parity))) return true;
  uint64_t t0 = global_ns();
  for (int spins = 1;; ++spins) {
    if (__all_sync(full, mbar_try_wait(bar, parity))) return true;
    if ((spins & 31) == 0) {
      if (__shfl_sync(full, *abort_flag, 0)) return false;
      const bool late = __shfl_sync(full, (global_ns() - t0) > kWaitLimitNs ? 1 : 0, 0);
      if (late) {
        if ((threadIdx.x & 31) == 0) {
          *abort_flag = 1;
          atomicOr(status, kStatusTimeout);
        }
        __syncwarp();
        return false;
      }
    }
  }
}

// Number of listed blocks of a tile and a pointer to its list (dense: implicit 0..i).
template <bool DENSE>
__device__ __forceinline__ int tile_len(const BsaParams& p, const Tile& t, const int32_t** list) {
  if (DENSE) {
    *list = nullptr;
    return t.i + 1;
  }
  const SeqInfo& s = p.bt.seq[t.b];
  const int row = s.row0 + t.i;
  const int beg = p.row_ptr[row];
  const int n = p.row_ptr[row + 1] - beg;
  *list = p.col_idx + static_cast<long long>(t.h) * p.bt.nnz_per_head + beg;
  return (n >= 1 && n <= t.i + 1) ? n : 0;
}

template <int D, int BN, bool FP8, bool PAGED, bool DENSE>
__global__ void __launch_bounds__(kThreads, 1) bsa_kernel(const __grid_constant__ BsaParams p) {
  using C = Cfg<D, BN, FP8>;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t sQ = sbase + C::OFF_Q;
  const uint32_t sK = sbase + C::OFF_K;
  const uint32_t sV = sbase + C::OFF_V;
  unsigned char* bar_area = smem + C::OFF_BAR;
  float* xch = reinterpret_cast<float*>(smem + C::OFF_XCH);
  // barriers (8 bytes each)
  const uint32_t b0 = sbase + C::OFF_BAR;
  const uint32_t bar_q_full = b0 + 0, bar_q_empty = b0 + 8;
  const uint32_t bar_k_full = b0 + 16, bar_k_empty = b0 + 48;   // [4]
  const uint32_t bar_v_full = b0 + 80, bar_v_empty = b0 + 112;  // [4]
  const uint32_t bar_s_full = b0 + 144;                         // [2]
  const uint32_t bar_p_full = b0 + 160, bar_pv_done = b0 + 168;
  const uint32_t bar_drain = b0 + 176, bar_x = b0 + 184;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_area + 256);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bar_area + 264);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  if (threadIdx.x == 0) {
    mbar_init(bar_q_full, 1);
    mbar_init(bar_q_empty, 1);
    for (int s = 0; s < C::KST; ++s) {
      mbar_init(bar_k_full + 8 * s, 1);
      mbar_init(bar_k_empty + 8 * s, 1);
    }
    for (int s = 0; s < C::VST; ++s) {
      mbar_init(bar_v_full + 8 * s, 1);
      mbar_init(bar_v_empty + 8 * s, 1);
    }
    mbar_init(bar_s_full, 1);
    mbar_init(bar_s_full + 8, 1);
    mbar_init(bar_p_full, kSoftmaxWarps);
    mbar_init(bar_pv_done, 1);
    mbar_init(bar_drain, 1);
    mbar_init(bar_x, kSoftmaxWarps);
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tmem_S = tmem;          // two S buffers at columns 0 and 128 (P overwrites S)
  const uint32_t tmem_O = tmem + 256;    // O of half 0 at 256, of half 1 at 256 + D

  const int G = p.Hq / p.Hkv;
  const unsigned full = 0xffffffffu;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_map(&p.tq);
      tma_prefetch_map(&p.tk);
      tma_prefetch_map(&p.tv);
    }
    uint32_t itk = 0, itv = 0, tq = 0;
    bool alive = true;
    for (int t = blockIdx.x; t < p.total_tiles && alive; t += gridDim.x) {
      const Tile tl = decode_tile(p, t);
      const int32_t* list;
      const int n = tile_len<DENSE>(p, tl, &list);
      if (n == 0) {
        if (lane == 0) atomicOr(p.status, kStatusBounds);
        continue;
      }
      const SeqInfo& s = p.bt.seq[tl.b];
      const int kvh = tl.h / G;
      if (!warp_wait(bar_q_empty, (tq & 1) ^ 1, abort_flag, p.status)) { alive = false; break; }
      if (lane == 0) {
        mbar_arrive_expect_tx(bar_q_full, C::Q_BYTES);
        for (int c = 0; c < C::DCH; ++c)
          tma_load_3d(sQ + c * C::Q_CHUNK, &p.tq, bar_q_full, c * C::CH, tl.h, s.tok0 + tl.i * BN);
      }
      ++tq;
      const int npages = (s.len + STEM_PAGE_SIZE - 1) / STEM_PAGE_SIZE;
      for (int j0 = 0; j0 < n && alive; j0 += 32) {
        const int jl = j0 + lane;
        int myj = jl;
        if (!DENSE) myj = jl < n ? __ldg(list + jl) : 0;
        if (jl < n && (myj < 0 || myj > tl.i)) {
          atomicOr(p.status, kStatusBounds);
          myj = tl.i;
        }
        if (jl >= n) myj = 0;
        // rows of this lane's block (one per 64-row box), resolved through the block table
        int rowh[C::HALVES];
#pragma unroll
        for (int hh = 0; hh < C::HALVES; ++hh) {
          if (PAGED) {
            int pg = (myj * BN) / STEM_PAGE_SIZE + hh;
            pg = pg < npages ? pg : npages - 1;
            int slot = (jl < n) ? __ldg(p.block_table + static_cast<long long>(tl.b) * p.max_pages + pg) : 0;
            if (slot < 0 || slot >= p.num_slots) {
              atomicOr(p.status, kStatusBounds);
              slot = 0;
            }
            rowh[hh] = slot * STEM_PAGE_SIZE;
          } else {
            rowh[hh] = s.tok0 + myj * BN + hh * 64;
          }
        }
        const int cnt = min(32, n - j0);
        for (int q = 0; q < cnt; ++q) {
          int rows[C::HALVES];
#pragma unroll
          for (int hh = 0; hh < C::HALVES; ++hh) rows[hh] = __shfl_sync(full, rowh[hh], q);
          const uint32_t ks = itk % C::KST, kph = (itk / C::KST) & 1;
          if (!warp_wait(bar_k_empty + 8 * ks, kph ^ 1, abort_flag, p.status)) { alive = false; break; }
          const bool withhold = p.inject == 1 && blockIdx.x == 0 && itk == 0;
          if (lane == 0 && !withhold) {
            mbar_arrive_expect_tx(bar_k_full + 8 * ks, C::KV_BYTES);
            for (int c = 0; c < C::DCH; ++c)
              for (int hh = 0; hh < C::HALVES; ++hh)
                tma_load_3d(sK + ks * C::KV_BYTES + c * C::KV_CHUNK + hh * 64 * 128, &p.tk, bar_k_full + 8 * ks,
                            c * C::CH, kvh, rows[hh]);
          }
          ++itk;
          const uint32_t vs = itv % C::VST, vph = (itv / C::VST) & 1;
          if (!warp_wait(bar_v_empty + 8 * vs, vph ^ 1, abort_flag, p.status)) { alive = false; break; }
          if (lane == 0) {
            mbar_arrive_expect_tx(bar_v_full + 8 * vs, C::KV_BYTES);
            for (int c = 0; c < C::DCH; ++c)
              for (int hh = 0; hh < C::HALVES; ++hh)
                tma_load_3d(sV + vs * C::KV_BYTES + c * C::KV_CHUNK + hh * 64 * 128, &p.tv, bar_v_full + 8 * vs,
                            c * C::CH, kvh, rows[hh]);
          }
          ++itv;
        }
      }
    }
    if (!alive) {
      // let the copies already issued land before the CTA can exit
      for (uint32_t q = (itk > C::KST ? itk - C::KST : 0); q < itk; ++q)
        for (int spin = 0; spin < 1000000 && !mbar_try_wait(bar_k_full + 8 * (q % C::KST), (q / C::KST) & 1); ++spin) {}
      for (uint32_t q = (itv > C::VST ? itv - C::VST : 0); q < itv; ++q)
        for (int spin = 0; spin < 1000000 && !mbar_try_wait(bar_v_full + 8 * (q % C::VST), (q / C::VST) & 1); ++spin) {}
      if (tq > 0)
        for (int spin = 0; spin < 1000000 && !mbar_try_wait(bar_q_full, (tq - 1) & 1); ++spin) {}
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    uint32_t itk = 0, itv = 0, is = 0, ip = 0, tq = 0;
    bool alive = true;
    auto issue_s = [&](void) -> bool {
      const uint32_t sb = is % 2;
      const uint32_t ks = itk % C::KST, kph = (itk / C::KST) & 1;
      if (!warp_wait(bar_k_full + 8 * ks, kph, abort_flag, p.status)) return false;
      tc_fence_after();
      if (lane == 0) {
#pragma unroll
        for (int k = 0; k < C::S_KSTEPS; ++k) {
          const int c = k / 4, w = k % 4;
          const uint64_t ad = smem_desc_sw128(sQ + c * C::Q_CHUNK + w * 32, 16, 1024);
          const uint64_t bd = smem_desc_sw128(sK + ks * C::KV_BYTES + c * C::KV_CHUNK + w * 32, 16, 1024);
          if (FP8)
            mma_fp8(tmem_S + sb * 128, ad, bd, C::IDESC_S, k > 0);
          else
            mma_bf16(tmem_S + sb * 128, ad, bd, C::IDESC_S, k > 0);
        }
        mma_commit(bar_s_full + 8 * sb);
        mma_commit(bar_k_empty + 8 * ks);
      }
      __syncwarp();
      ++is;
      ++itk;
      return true;
    };
    for (int t = blockIdx.x; t < p.total_tiles && alive; t += gridDim.x) {
      const Tile tl = decode_tile(p, t);
      const int32_t* list;
      const int n = tile_len<DENSE>(p, tl, &list);
      if (n == 0) continue;
      if (!warp_wait(bar_q_full, tq & 1, abort_flag, p.status)) { alive = false; break; }
      ++tq;
      if (!issue_s()) { alive = false; break; }
      for (int jj = 0; jj < n; ++jj) {
        if (jj + 1 < n) {
          if (!issue_s()) { alive = false; break; }
        }
        if (jj + 1 == n) {
          if (lane == 0) mma_commit(bar_q_empty);  // all S MMAs of the tile issued
          __syncwarp();
        }
        const uint32_t pb = ip % 2;
        if (!warp_wait(bar_p_full, ip & 1, abort_flag, p.status)) { alive = false; break; }
        ++ip;
        const uint32_t vs = itv % C::VST, vph = (itv / C::VST) & 1;
        if (!warp_wait(bar_v_full + 8 * vs, vph, abort_flag, p.status)) { alive = false; break; }
        tc_fence_after();
        if (lane == 0) {
#pragma unroll
          for (int k = 0; k < C::PV_KSTEPS; ++k) {
            // half hf of the block's keys: its P (in that half's S columns) into its own O
            const int hf = k / C::PV_HSTEPS, kk = k % C::PV_HSTEPS;
            const uint64_t bd =
                smem_desc_sw128(sV + vs * C::KV_BYTES + k * C::PV_KROWS * 128, C::KV_CHUNK, 1024);
            const uint32_t a_tmem = tmem_S + pb * 128 + hf * C::HALF + kk * 8;
            const uint32_t d_tmem = tmem_O + hf * D;
            const uint32_t acc = (jj > 0 || kk > 0) ? 1u : 0u;
            if (FP8)
              mma_fp8_ts(d_tmem, a_tmem, bd, C::IDESC_PV, acc);
            else
              mma_bf16_ts(d_tmem, a_tmem, bd, C::IDESC_PV, acc);
          }
          mma_commit(bar_v_empty + 8 * vs);
          mma_commit(bar_pv_done);
        }
        __syncwarp();
        ++itv;
      }
    }
    // drain: every tcgen05.mma issued by this thread has completed
    if (lane == 0) mma_commit(bar_drain);
    __syncwarp();
    for (int spin = 0; spin < 4000000 && !mbar_try_wait(bar_drain, 0); ++spin) {}
  } else {
    // ------------------------------------------------------------ softmax + epilogue
    const int wg = (warp - 2) / 4;                   // which half of the KV block's columns
    const int quad = warp % 4;                       // TMEM lane quadrant of this warp
    const int r = quad * 32 + lane;                  // query row within the tile
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t my_O = tmem_O + wg * D + lane_off;
    const float sl2 = p.scale_log2;
    uint32_t gb = 0, ix = 0;                         // blocks processed by this CTA; exchanges
    bool alive = true;
    for (int t = blockIdx.x; t < p.total_tiles && alive; t += gridDim.x) {
      const Tile tl = decode_tile(p, t);
      const int32_t* list;
      const int n = tile_len<DENSE>(p, tl, &list);
      if (n == 0) continue;
      // per half: running max, sum of the rounded P the product uses (normalises O) and,
      // for FP8, the sum of the unrounded P (log-sum-exp)
      float m_run = -INFINITY;
      float2 l2 = make_float2(0.f, 0.f), lt2 = make_float2(0.f, 0.f);
      for (int jj = 0; jj < n; ++jj, ++gb) {
        const uint32_t sb = gb % 2, sph = (gb / 2) & 1;
        if (!warp_wait(bar_s_full + 8 * sb, sph, abort_flag, p.status)) { alive = false; break; }
        tc_fence_after();
        const uint32_t my_S = tmem_S + sb * 128 + wg * C::HALF + lane_off;
        uint32_t sr[C::HALF];
#pragma unroll
        for (int c = 0; c < C::HALF / 32; ++c) tmem_ld32(my_S + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[c * 32]));
        tmem_wait_ld();
        const bool diag = (jj == n - 1);
        if (diag) {
#pragma unroll
          for (int c = 0; c < C::HALF; ++c)
            if (wg * C::HALF + c > r) sr[c] = __float_as_uint(-INFINITY);
        }
        // row maximum with four independent chains
        float mq[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int c = 0; c < C::HALF; c += 8)
#pragma unroll
          for (int q = 0; q < 4; ++q) mq[q] = max3f(mq[q], __uint_as_float(sr[c + 2 * q]), __uint_as_float(sr[c + 2 * q + 1]));
        const float mx = fmaxf(max3f(mq[0], mq[1], mq[2]), mq[3]);
        const float m_new = fmaxf(m_run, mx * sl2);
        const bool resc = m_new > m_run + 8.0f;
        const float m_use = resc ? m_new : m_run;
        const float alpha = resc ? ex2_approx(m_run - m_use) : 1.0f;
        const float2 sc2 = make_float2(sl2, sl2);
        // a half that has seen only masked keys so far (m = -inf) gets P = 0, not NaN
        const float m_sub = m_use == -INFINITY ? 0.f : m_use;
        const float2 bias2 = make_float2(p.p_bias - m_sub, p.p_bias - m_sub);
        // sums with four independent chains
        float2 sq[4], tq4[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          sq[q] = make_float2(0.f, 0.f);
          tq4[q] = make_float2(0.f, 0.f);
        }
        uint32_t pk[C::P_COLS];
        if (!FP8) {
#pragma unroll
          for (int u = 0; u < C::HALF / 2; ++u) {
            const float2 y = fma2(make_float2(__uint_as_float(sr[2 * u]), __uint_as_float(sr[2 * u + 1])), sc2, bias2);
            const uint32_t w = pack_bf16x2(ex2_approx(y.x), ex2_approx(y.y));
            pk[u] = w;
            sq[u % 4] = add2(sq[u % 4], make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u)));
          }
        } else {
          // e4m3 P; its rounded values are summed as f16 pairs (exact enough: two e4m3
          // codes per f16 add) and the unrounded values only when the LSE is requested
          auto fp8_block = [&](auto want_lse) {
#pragma unroll
            for (int u = 0; u < C::HALF / 4; ++u) {
              const float2 y0 = fma2(make_float2(__uint_as_float(sr[4 * u]), __uint_as_float(sr[4 * u + 1])), sc2, bias2);
              const float2 y1 = fma2(make_float2(__uint_as_float(sr[4 * u + 2]), __uint_as_float(sr[4 * u + 3])), sc2, bias2);
              const float2 e0 = make_float2(ex2_approx(y0.x), ex2_approx(y0.y));
              const float2 e1 = make_float2(ex2_approx(y1.x), ex2_approx(y1.y));
              const uint32_t lo = pack_e4m3x2(e0.x, e0.y);
              const uint32_t hi = pack_e4m3x2(e1.x, e1.y);
              pk[u] = __byte_perm(lo, hi, 0x5410);
              sq[u % 4] = add2(sq[u % 4], e4m3x4_pairsum(pk[u]));
              if constexpr (decltype(want_lse)::value) tq4[u % 4] = add2(tq4[u % 4], add2(e0, e1));
            }
          };
          if (p.lse != nullptr)
            fp8_block(std::true_type{});
          else
            fp8_block(std::false_type{});
        }
        const float2 sum2 = add2(add2(sq[0], sq[1]), add2(sq[2], sq[3]));
        const float2 sumt2 = add2(add2(tq4[0], tq4[1]), add2(tq4[2], tq4[3]));
        // P overwrites the first columns of this half's S, packed along columns
        static_assert(C::P_COLS == 32 || C::P_COLS == 16, "P columns per half");
        if constexpr (C::P_COLS == 32)
          tmem_st32(my_S, *reinterpret_cast<uint32_t(*)[32]>(&pk[0]));
        else
          tmem_st16(my_S, &pk[0]);
        const float2 a2 = make_float2(alpha, alpha);
        l2 = fma2(l2, a2, sum2);
        if (FP8) lt2 = fma2(lt2, a2, sumt2);
        if (jj > 0 && __any_sync(full, resc)) {
          // O of this half holds the sum up to the previous block once its P V product is
          // done (the barrier cannot be two phases ahead: the next product needs this warp)
          if (!warp_wait(bar_pv_done, (gb - 1) & 1, abort_flag, p.status)) { alive = false; break; }
          tc_fence_after();
#pragma unroll
          for (int c = 0; c < D / 16; ++c) {
            uint32_t o[16];
            tmem_ld16(my_O + c * 16, o);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 16; e += 2) {
              const float2 v = mul2(make_float2(__uint_as_float(o[e]), __uint_as_float(o[e + 1])), a2);
              o[e] = __float_as_uint(v.x);
              o[e + 1] = __float_as_uint(v.y);
            }
            tmem_st16(my_O + c * 16, o);
          }
        }
        tmem_wait_st();
        m_run = m_use;
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_p_full);
      }
      if (!alive) break;
      // epilogue: wait for the last P V product, merge the two halves, normalise, store
      if (!warp_wait(bar_pv_done, (gb - 1) & 1, abort_flag, p.status)) { alive = false; break; }
      tc_fence_after();
      float* mine = xch + wg * 128 + r;
      mine[0] = m_run;
      mine[256] = l2.x + l2.y;
      mine[512] = lt2.x + lt2.y;
      __syncwarp();
      if (lane == 0) {
        __threadfence_block();
        mbar_arrive(bar_x);
      }
      if (!warp_wait(bar_x, ix & 1, abort_flag, p.status)) { alive = false; break; }
      ++ix;
      const float m0 = xch[r], m1 = xch[128 + r];
      const float l0 = xch[256 + r], l1 = xch[384 + r];
      const float t0 = xch[512 + r], t1 = xch[640 + r];
      const float mf = fmaxf(m0, m1);
      const float f0 = ex2_approx(m0 - mf), f1 = ex2_approx(m1 - mf);
      const float l = l0 * f0 + l1 * f1;
      const float inv = p.out_scale / l;
      const float g0 = f0 * inv, g1 = f1 * inv;
      const SeqInfo& s = p.bt.seq[tl.b];
      const int rows_valid = min(BN, s.len - tl.i * BN);
      const long long tok = static_cast<long long>(s.tok0) + tl.i * BN + r;
      unsigned char* orow = static_cast<unsigned char*>(p.out) + ((tok * p.Hq + tl.h) * D + wg * C::O_HALF) * 2;
      const float2 gg0 = make_float2(g0, g0), gg1 = make_float2(g1, g1);
#pragma unroll
      for (int c = 0; c < C::O_HALF / 16; ++c) {
        uint32_t oa[16], ob[16];
        tmem_ld16(tmem_O + wg * C::O_HALF + lane_off + c * 16, oa);
        tmem_ld16(tmem_O + D + wg * C::O_HALF + lane_off + c * 16, ob);
        tmem_wait_ld();
        if (r < rows_valid) {
          uint32_t w[8];
#pragma unroll
          for (int e = 0; e < 16; e += 2) {
            const float2 v = fma2(make_float2(__uint_as_float(oa[e]), __uint_as_float(oa[e + 1])), gg0,
                                  mul2(make_float2(__uint_as_float(ob[e]), __uint_as_float(ob[e + 1])), gg1));
            w[e / 2] = pack_bf16x2(v.x, v.y);
          }
          *reinterpret_cast<uint4*>(orow + c * 32) = make_uint4(w[0], w[1], w[2], w[3]);
          *reinterpret_cast<uint4*>(orow + c * 32 + 16) = make_uint4(w[4], w[5], w[6], w[7]);
        }
      }
      if (p.lse != nullptr && wg == 0 && r < rows_valid) {
        const float lt = FP8 ? (t0 * f0 + t1 * f1) / p.p_scale : l;
        p.lse[static_cast<long long>(tl.h) * p.bt.total_tokens + tok] = (mf + __log2f(lt)) * 0.69314718055994531f;
      }
      tc_fence_before();
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, kTmemCols);
}

// ------------------------------------------------------------------ host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode() {
  static EncodeTiledFn fn = nullptr;
  if (fn == nullptr) {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &f, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(f);
  }
  return fn;
}

// 3-D map over a token-major [rows, H, d] tensor: dims (d, H, rows), box (box_d, 1, box_rows).
bool make_map(CUtensorMap* m, const void* ptr, bool fp8, int d, int H, long long rows, int box_d, int box_rows) {
  EncodeTiledFn enc = get_encode();
  if (enc == nullptr) return false;
  const int es = fp8 ? 1 : 2;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * es, static_cast<cuuint64_t>(H) * d * es};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(box_d), 1u, static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[3] = {1u, 1u, 1u};
  CUresult r = enc(m, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
                   const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int D, int BN, bool FP8, bool PAGED, bool DENSE>
cudaError_t run(const BsaParams& prm, cudaStream_t st) {
  using C = Cfg<D, BN, FP8>;
  auto kern = bsa_kernel<D, BN, FP8, PAGED, DENSE>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_LAUNCH);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int grid = prm.total_tiles < sms ? prm.total_tiles : sms;
  if (grid <= 0) return cudaSuccess;
  kern<<<grid, kThreads, C::SMEM_LAUNCH, st>>>(prm);
  return cudaGetLastError();
}

template <int D, int BN, bool FP8>
cudaError_t run_mode(const BsaParams& prm, bool paged, bool dense, cudaStream_t st) {
  if (paged) return dense ? run<D, BN, FP8, true, true>(prm, st) : run<D, BN, FP8, true, false>(prm, st);
  return dense ? run<D, BN, FP8, false, true>(prm, st) : run<D, BN, FP8, false, false>(prm, st);
}

}  // namespace

cudaError_t launch_bsa(const Batch& bt, const BsaArgs& a, bool fp8, bool paged, bool dense, uint32_t* status,
                       cudaStream_t st) {
  BsaParams prm;
  memset(&prm, 0, sizeof(prm));
  const int D = a.head_dim, BN = bt.block;
  const int ch = fp8 ? 128 : 64;
  const int box_d = D < ch ? D : ch;
  if (!make_map(&prm.tq, a.q, fp8, D, a.Hq, bt.total_tokens, box_d, kBM)) return cudaErrorInvalidValue;
  if (!make_map(&prm.tk, a.k, fp8, D, a.Hkv, a.kv_rows, box_d, 64)) return cudaErrorInvalidValue;
  if (!make_map(&prm.tv, a.v, fp8, D, a.Hkv, a.kv_rows, box_d, 64)) return cudaErrorInvalidValue;
  prm.bt = bt;
  prm.row_ptr = a.row_ptr;
  prm.col_idx = a.col_idx;
  prm.block_table = a.block_table;
  prm.max_pages = a.max_pages;
  prm.num_slots = paged ? static_cast<int>(a.kv_rows / STEM_PAGE_SIZE) : 0;
  prm.out = a.out;
  prm.lse = a.lse;
  prm.Hq = a.Hq;
  prm.Hkv = a.Hkv;
  prm.status = status;
  prm.inject = take_injection();
  const float log2e = 1.4426950408889634f;
  prm.scale_log2 = a.sigma * (fp8 ? a.q_scale * a.k_scale : 1.0f) * log2e;
  // FP8: P <= 2^8 after the lazy max update; 448 / 256 keeps it inside e4m3's range.
  prm.p_scale = fp8 ? 1.75f : 1.0f;
  prm.p_bias = fp8 ? 0.80735492205760410f : 0.0f;  // log2(1.75)
  // l is accumulated from the scaled, rounded P, so the V scale is all that remains
  prm.out_scale = fp8 ? a.v_scale : 1.0f;
  long long tiles = 0;
  for (int b = 0; b < bt.num_seqs; ++b) tiles += static_cast<long long>(bt.seq[b].nblk) * a.Hq;
  prm.total_tiles = static_cast<int>(tiles);
  // sequences by decreasing block count (longest rows first)
  int ord[STEM_MAX_SEQS];
  for (int b = 0; b < bt.num_seqs; ++b) ord[b] = b;
  for (int x = 1; x < bt.num_seqs; ++x)
    for (int y = x; y > 0 && bt.seq[ord[y]].nblk > bt.seq[ord[y - 1]].nblk; --y) {
      int tmp = ord[y];
      ord[y] = ord[y - 1];
      ord[y - 1] = tmp;
    }
  for (int b = 0; b < bt.num_seqs; ++b) prm.order[b] = static_cast<signed char>(ord[b]);

  if (fp8) {
    if (D == 128 && BN == 128) return run_mode<128, 128, true>(prm, paged, dense, st);
    return cudaErrorInvalidValue;
  }
  if (D == 128 && BN == 128) return run_mode<128, 128, false>(prm, paged, dense, st);
  if (D == 128 && BN == 64) return run_mode<128, 64, false>(prm, paged, dense, st);
  if (D == 64 && BN == 128) return run_mode<64, 128, false>(prm, paged, dense, st);
  if (D == 64 && BN == 64) return run_mode<64, 64, false>(prm, paged, dense, st);
  return cudaErrorInvalidValue;
}

}  // namespace stem
