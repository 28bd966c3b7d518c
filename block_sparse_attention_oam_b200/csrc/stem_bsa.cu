// Block-sparse causal flash-attention prefill on sm_100a (tcgen05 + TMEM + TMA).
//
// Tencent Cloud article "从Stem稀疏注意力看 大模型推理的架构取舍", section
// "HPC-BSA：跳块零开销的秘密": for each Q block the kernel holds the list of KV
// blocks to visit and its inner loop walks only that list, with no per-block
// "skip?" branch; a skipped block is mathematically the same as all its scores
// being -inf, so the softmax stays exact; the inner path is the dense one.  The
// same section notes native support for a paged KV cache.
//
// Design (one CTA per SM, persistent, 10 warps).  Work unit: one q-block row i of one
// sequence for a PAIR of q-heads (2p, 2p+1).  Both tiles of a pair list the same number of
// blocks (the budget k_i does not depend on the head), so they advance in lock-step in
// two "slots" that share the tensor core (ping-pong): while the softmax of one slot works
// on its scores, the tensor core runs the other slot's P V and next S.
//   warp 0      TMA producer: per slot, the Q tile once per unit, then K_j and V_j of
//               every listed block into per-slot rings (64-row boxes, 128-byte swizzle;
//               a paged cache is read page by page through the block table).
//   warp 1      MMA issuer (one thread): per slot, S = Q K_j^T into the slot's TMEM S/P
//               columns, then O += P_j V_j with P read from TMEM (where the softmax wrote
//               it over S_j) and V from shared memory.  Order per block j:
//               PV_0(j), S_0(j+1), PV_1(j), S_1(j+1).
//   warps 2..5  softmax of slot 0, warps 6..9 softmax of slot 1: one thread per query row
//               (TMEM lane quadrant = warp % 4).  Online softmax in the log2 domain with
//               packed fp32x2 arithmetic; the token-level causal mask only on the diagonal
//               block (always the last list entry); O rescaled lazily (only when the
//               running max grows by more than 2^8) — no wait is needed for that, since
//               S_j is issued after P V_{j-1} and the tensor core runs in order; O
//               normalised by the sum of the P weights (BF16: as rounded for the product;
//               FP8: unrounded, except on a sequence's first row); then the epilogue
//               (O / l -> bf16, log-sum-exp).
// Every wait is bounded (2 s); on expiry the CTA raises an abort flag, records
// STEM_ERR_TIMEOUT in the status word, drains its tensor-core work, waits (bounded)
// for its copies and releases its TMEM before exiting.
#include <string.h>

#include <type_traits>

#include "stem_internal.cuh"

namespace stem {
namespace {

constexpr int kBM = 128;              // query rows per tile (tcgen05 M)
constexpr int kThreads = 64 + 256;    // producer, MMA, two softmax warpgroups
constexpr uint32_t kTmemCols = 512;   // per slot: S/P at +0 (128 columns), O at +128 (D)
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
  static constexpr int P_COLS = BN * ES / 4;      // TMEM columns of a row's P (packed)
  static constexpr int EXTRA = 512;               // barriers and flags
  static constexpr int SLACK = 1024;              // alignment of the tiles to 1024 bytes
  // per-slot K and V ring depth: as deep as shared memory allows, at most 4
  static constexpr int ROOM = static_cast<int>(kSmemCap) - 2 * Q_BYTES - EXTRA - SLACK;
  static constexpr int NST0 = ROOM / (4 * KV_BYTES);
  static constexpr int NST = NST0 > 4 ? 4 : (NST0 < 1 ? 1 : NST0);
  static_assert(4 * NST * KV_BYTES <= ROOM, "K/V rings do not fit");
  static constexpr int OFF_Q = 0;                               // [slot]
  static constexpr int OFF_K = 2 * Q_BYTES;                     // [slot][stage]
  static constexpr int OFF_V = OFF_K + 2 * NST * KV_BYTES;      // [slot][stage]
  static constexpr int OFF_BAR = OFF_V + 2 * NST * KV_BYTES;
  static constexpr int SMEM = OFF_BAR + EXTRA + SLACK;
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
  int list_group;    // q-heads per list (1, or Hq/Hkv with shared lists)
  const int32_t* block_table;
  int max_pages;
  int num_slots;
  void* out;
  float* lse;
  int Hq, Hkv;
  int total_units;   // sum over sequences of N_b * ceil(Hq / 2)
  int groups;        // (sequence, head pair) groups with at least one unit in this launch
  float scale_log2;  // sigma * q_scale * k_scale * log2(e)
  float p_bias;      // log2 of the factor P is scaled by before rounding (FP8: log2 1.75)
  float out_scale;   // FP8: v_scale (l carries the P factor); BF16: 1
  float p_scale;     // the factor itself (1 for BF16)
  uint32_t* status;
  int inject;        // 1: CTA 0 withholds its first K tile (failure-detection test)
  signed char order[STEM_MAX_SEQS];  // sequences by decreasing block count
};

struct Unit {
  int b, i, h0;      // sequence, q-block row, first q-head of the pair
  bool two;          // the pair's second head exists
};

// Which units a launch covers.  kAllRows: every q-block row.  kRestRows: rows 1..N-1 of
// every sequence; kFirstRow: row 0 only (FP8 runs the two, the first-row launch with the
// two-term P; see the softmax).
enum : int { kAllRows = 0, kRestRows = 1, kFirstRow = 2 };

// Unit order: sequences by decreasing length; inside a sequence head pair by head pair,
// so that the CTAs running at one time share one pair's kv-head(s), whose K/V fit in L2.
// The rows of a group run alternately from the last (longest list) to the first and back,
// the final group longest first: list lengths then change smoothly from unit to unit, and
// the round-robin split over the CTAs gives each nearly the same number of blocks (a row
// order that restarts at the longest row in every group leaves the first CTAs with the
// longest row of every round).
template <int PART>
__device__ __forceinline__ Unit decode_unit(const BsaParams& p, int u) {
  Unit r{0, 0, 0, false};
  const int NP = (p.Hq + 1) / 2;
  int acc = 0;
  for (int q = 0; q < p.bt.num_seqs; ++q) {
    const int b = p.order[q];
    const int nb = PART == kFirstRow ? 1 : (PART == kRestRows ? p.bt.seq[b].nblk - 1 : p.bt.seq[b].nblk);
    const int nu = nb * NP;
    if (u < acc + nu) {
      const int local = u - acc;
      const int pair = local / nb;
      const int pos = local - pair * nb;
      const bool longest_first = ((p.groups - 1 - (q * NP + pair)) & 1) == 0;
      r.b = b;
      r.i = PART == kFirstRow ? 0 : (longest_first ? p.bt.seq[b].nblk - 1 - pos : p.bt.seq[b].nblk - nb + pos);
      r.h0 = 2 * pair;
      r.two = r.h0 + 1 < p.Hq;
      return r;
    }
    acc += nu;
  }
  return r;
}

// The CTAs take the units round robin (CTA c: c, c + gridDim, ...).  With an odd number
// of groups the last one has no partner running the other way (a single head pair:
// nothing cancels, and CTA 0 gets the longest row of every round, 12 % above the mean at
// 128K); those launches (the SNAKE kernels) deal every window of 2 x gridDim units
// forwards and back instead, so that each CTA pairs a longer row with a shorter one
// (1.6 % at 128K; three pairs 4 % -> 1.3 %).  snake_unit: the CTA's k-th unit, or
// total_units when it has none left.
__device__ __forceinline__ int snake_unit(const BsaParams& p, int k) {
  const int g = static_cast<int>(gridDim.x), c = static_cast<int>(blockIdx.x), base = (k >> 1) * 2 * g;
  if ((k & 1) == 0) return min(base + c, p.total_units);
  const int len = min(2 * g, p.total_units - base);
  return c < len - g ? base + len - 1 - c : p.total_units;
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

// Number of listed blocks of a row (the same for every head) and a head's list
// (dense: implicit 0..i).
template <bool DENSE>
__device__ __forceinline__ int unit_len(const BsaParams& p, const Unit& un) {
  if (DENSE) return un.i + 1;
  const int row = p.bt.seq[un.b].row0 + un.i;
  const int n = p.row_ptr[row + 1] - p.row_ptr[row];
  return (n >= 1 && n <= un.i + 1) ? n : 0;
}
__device__ __forceinline__ const int32_t* head_list(const BsaParams& p, const Unit& un, int h) {
  const int row = p.bt.seq[un.b].row0 + un.i;
  return p.col_idx + static_cast<long long>(h / p.list_group) * p.bt.nnz_per_head + p.row_ptr[row];
}

template <int D, int BN, bool FP8, bool PAGED, bool DENSE, int PART, bool SHKV, bool LSEX, bool SNAKE>
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
  // per-slot barriers (8 bytes each), slot s at b0 + 192 s
  const uint32_t b0 = sbase + C::OFF_BAR;
  auto q_full = [&](int s) { return b0 + 192 * s + 0; };
  auto q_empty = [&](int s) { return b0 + 192 * s + 8; };
  auto k_full = [&](int s, int t) { return b0 + 192 * s + 16 + 8 * t; };
  auto k_empty = [&](int s, int t) { return b0 + 192 * s + 48 + 8 * t; };
  auto v_full = [&](int s, int t) { return b0 + 192 * s + 80 + 8 * t; };
  auto v_empty = [&](int s, int t) { return b0 + 192 * s + 112 + 8 * t; };
  auto s_full = [&](int s) { return b0 + 192 * s + 144; };
  auto p_full = [&](int s) { return b0 + 192 * s + 152; };
  auto o_done = [&](int s) { return b0 + 192 * s + 160; };
  const uint32_t bar_drain = b0 + 384;
  // K/V rings.  Per slot: NST stages each.  SHKV (both tiles of a pair walk one list of one
  // kv-head): one ring of 2*NST stages over both slots' memory, each tile loaded once and
  // released after both slots' products (empty barriers expect two arrivals).
  constexpr int RING = SHKV ? 2 * C::NST : C::NST;
  auto kv_off = [&](int s, uint32_t t) { return (SHKV ? t : s * C::NST + t) * C::KV_BYTES; };
  auto kf = [&](int s, uint32_t t) { return SHKV ? k_full(t / C::NST, t % C::NST) : k_full(s, t); };
  auto ke = [&](int s, uint32_t t) { return SHKV ? k_empty(t / C::NST, t % C::NST) : k_empty(s, t); };
  auto vf = [&](int s, uint32_t t) { return SHKV ? v_full(t / C::NST, t % C::NST) : v_full(s, t); };
  auto ve = [&](int s, uint32_t t) { return SHKV ? v_empty(t / C::NST, t % C::NST) : v_empty(s, t); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_area + 448);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bar_area + 456);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(q_full(s), 1);
      mbar_init(q_empty(s), 1);
      for (int t = 0; t < C::NST; ++t) {
        mbar_init(k_full(s, t), 1);
        mbar_init(k_empty(s, t), SHKV ? 2 : 1);
        mbar_init(v_full(s, t), 1);
        mbar_init(v_empty(s, t), SHKV ? 2 : 1);
      }
      mbar_init(s_full(s), 1);
      mbar_init(p_full(s), 4);
      mbar_init(o_done(s), 1);
    }
    mbar_init(bar_drain, 1);
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
  const int G = p.Hq / p.Hkv;
  const unsigned full = 0xffffffffu;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_map(&p.tq);
      tma_prefetch_map(&p.tk);
      tma_prefetch_map(&p.tv);
    }
    uint32_t itk[2] = {0, 0}, itv[2] = {0, 0}, tq = 0;
    bool alive = true;
    for (int k = 0, u = blockIdx.x; u < p.total_units && alive; u = SNAKE ? snake_unit(p, ++k) : u + gridDim.x) {
      const Unit un = decode_unit<PART>(p, u);
      const int n = unit_len<DENSE>(p, un);
      if (n == 0) {
        if (lane == 0) atomicOr(p.status, kStatusBounds);
        continue;
      }
      const int ns = un.two ? 2 : 1;
      const SeqInfo& sq = p.bt.seq[un.b];
      for (int s = 0; s < ns; ++s) {
        if (!warp_wait(q_empty(s), (tq & 1) ^ 1, abort_flag, p.status)) { alive = false; break; }
        if (lane == 0) {
          mbar_arrive_expect_tx(q_full(s), C::Q_BYTES);
          for (int c = 0; c < C::DCH; ++c)
            tma_load_3d(sQ + s * C::Q_BYTES + c * C::Q_CHUNK, &p.tq, q_full(s), c * C::CH, un.h0 + s,
                        sq.tok0 + un.i * BN);
        }
      }
      if (!alive) break;
      ++tq;
      const int npages = (sq.len + STEM_PAGE_SIZE - 1) / STEM_PAGE_SIZE;
      const int32_t* lists[2] = {DENSE ? nullptr : head_list(p, un, un.h0),
                                 DENSE || !un.two ? nullptr : head_list(p, un, un.h0 + 1)};
      for (int j0 = 0; j0 < n && alive; j0 += 32) {
        const int jl = j0 + lane;
        // rows of this lane's block for each slot (one per 64-row box)
        int rowh[2][C::HALVES];
#pragma unroll
        for (int s = 0; s < 2; ++s) {
          int myj = jl;
          if (!DENSE) myj = (jl < n && s < ns) ? __ldg(lists[s] + jl) : 0;
          // every entry lies in 0..i and the last one is the diagonal block (the only one
          // the token-level mask applies to); anything else is reported, and the diagonal
          // block read in its place
          if (jl < n && s < ns && (myj < 0 || myj > un.i || (jl == n - 1 && myj != un.i))) {
            atomicOr(p.status, kStatusBounds);
            myj = un.i;
          }
          if (jl >= n || s >= ns) myj = 0;
#pragma unroll
          for (int hh = 0; hh < C::HALVES; ++hh) {
            if (PAGED) {
              int pg = (myj * BN) / STEM_PAGE_SIZE + hh;
              pg = pg < npages ? pg : npages - 1;
              int slot = (jl < n && s < ns) ? __ldg(p.block_table + static_cast<long long>(un.b) * p.max_pages + pg) : 0;
              if (slot < 0 || slot >= p.num_slots) {
                atomicOr(p.status, kStatusBounds);
                slot = 0;
              }
              rowh[s][hh] = slot * STEM_PAGE_SIZE;
            } else {
              rowh[s][hh] = sq.tok0 + myj * BN + hh * 64;
            }
          }
        }
        const int cnt = min(32, n - j0);
        for (int q = 0; q < cnt && alive; ++q) {
          int rows[2][C::HALVES];
#pragma unroll
          for (int s = 0; s < 2; ++s)
#pragma unroll
            for (int hh = 0; hh < C::HALVES; ++hh) rows[s][hh] = __shfl_sync(full, rowh[s][hh], q);
          for (int s = 0; s < ns; ++s) {
            const int kvh = (un.h0 + s) / G;
            if (SHKV && s > 0) break;  // one copy of the shared tile
            const uint32_t t = itk[s] % RING, ph = (itk[s] / RING) & 1;
            if (!warp_wait(ke(s, t), ph ^ 1, abort_flag, p.status)) { alive = false; break; }
            const bool withhold = p.inject == 1 && blockIdx.x == 0 && s == 0 && itk[0] == 0;
            if (lane == 0 && !withhold) {
              mbar_arrive_expect_tx(kf(s, t), C::KV_BYTES);
              for (int c = 0; c < C::DCH; ++c)
                for (int hh = 0; hh < C::HALVES; ++hh)
                  tma_load_3d(sK + kv_off(s, t) + c * C::KV_CHUNK + hh * 64 * 128, &p.tk, kf(s, t), c * C::CH,
                              kvh, rows[s][hh]);
            }
            ++itk[s];
          }
          for (int s = 0; s < ns && alive; ++s) {
            const int kvh = (un.h0 + s) / G;
            if (SHKV && s > 0) break;
            const uint32_t t = itv[s] % RING, ph = (itv[s] / RING) & 1;
            if (!warp_wait(ve(s, t), ph ^ 1, abort_flag, p.status)) { alive = false; break; }
            if (lane == 0) {
              mbar_arrive_expect_tx(vf(s, t), C::KV_BYTES);
              for (int c = 0; c < C::DCH; ++c)
                for (int hh = 0; hh < C::HALVES; ++hh)
                  tma_load_3d(sV + kv_off(s, t) + c * C::KV_CHUNK + hh * 64 * 128, &p.tv, vf(s, t), c * C::CH,
                              kvh, rows[s][hh]);
            }
            ++itv[s];
          }
        }
      }
    }
    if (!alive) {
      // let the copies already issued land before the CTA can exit
      for (int s = 0; s < 2; ++s) {
        for (uint32_t q = (itk[s] > RING ? itk[s] - RING : 0); q < itk[s]; ++q)
          for (int spin = 0; spin < 1000000 && !mbar_try_wait(kf(s, q % RING), (q / RING) & 1); ++spin) {}
        for (uint32_t q = (itv[s] > RING ? itv[s] - RING : 0); q < itv[s]; ++q)
          for (int spin = 0; spin < 1000000 && !mbar_try_wait(vf(s, q % RING), (q / RING) & 1); ++spin) {}
      }
      if (tq > 0)
        for (int s = 0; s < 2; ++s)
          for (int spin = 0; spin < 1000000 && !mbar_try_wait(q_full(s), (tq - 1) & 1); ++spin) {}
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // One thread does all of it: its waits and commits then cost no warp-wide votes.
    if (lane == 0) {
      uint32_t itk[2] = {0, 0}, itv[2] = {0, 0}, gb[2] = {0, 0}, tq = 0;
      bool alive = true;
      // S = Q K^T of a block (K in ring stage t) into the slot's S/P columns
      auto issue_mmas_s = [&](int s, uint32_t t) {
        const uint32_t d_tmem = tmem + 256 * s;
#pragma unroll
        for (int k = 0; k < C::S_KSTEPS; ++k) {
          const int c = k / 4, w = k % 4;
          const uint64_t ad = smem_desc_sw128(sQ + s * C::Q_BYTES + c * C::Q_CHUNK + w * 32, 16, 1024);
          const uint64_t bd =
              smem_desc_sw128(sK + kv_off(s, t) + c * C::KV_CHUNK + w * 32, 16, 1024);
          if (FP8)
            mma_fp8(d_tmem, ad, bd, C::IDESC_S, k > 0);
          else
            mma_bf16(d_tmem, ad, bd, C::IDESC_S, k > 0);
        }
      };
      // the first S of a unit
      auto issue_s = [&](int s, bool last) -> bool {
        const uint32_t t = itk[s] % RING, ph = (itk[s] / RING) & 1;
        if (!mbar_wait(kf(s, t), ph, abort_flag, p.status)) return false;
        tc_fence_after();
        issue_mmas_s(s, t);
        mma_commit(s_full(s));
        mma_commit(ke(s, t));
        if (last) mma_commit(q_empty(s));  // every S of this unit issued: Q may be replaced
        ++itk[s];
        return true;
      };
      for (int k = 0, u = blockIdx.x; u < p.total_units && alive; u = SNAKE ? snake_unit(p, ++k) : u + gridDim.x) {
        const Unit un = decode_unit<PART>(p, u);
        const int n = unit_len<DENSE>(p, un);
        if (n == 0) continue;
        const int ns = un.two ? 2 : 1;
        for (int s = 0; s < ns && alive; ++s) {
          if (!mbar_wait(q_full(s), tq & 1, abort_flag, p.status)) { alive = false; break; }
          if (!issue_s(s, n == 1)) { alive = false; break; }
        }
        ++tq;
        for (int jj = 0; jj < n && alive; ++jj) {
          for (int s = 0; s < ns; ++s) {
            // With two or more ring stages, V_j and K_{j+1} have landed long before P_j is
            // ready: wait for them first, so that P V_j and S_{j+1} go out back to back as
            // soon as P_j arrives.  With one stage K_{j+1} is only loaded once S_j is done,
            // so P V_j goes first and the wait for K_{j+1} follows it.
            constexpr bool kEarlyK = RING >= 2;
            const uint32_t t = itv[s] % RING, ph = (itv[s] / RING) & 1;
            if (!mbar_wait(vf(s, t), ph, abort_flag, p.status)) { alive = false; break; }
            const bool more = jj + 1 < n;
            const uint32_t tk = itk[s] % RING, pk = (itk[s] / RING) & 1;
            if (kEarlyK && more && !mbar_wait(kf(s, tk), pk, abort_flag, p.status)) { alive = false; break; }
            if (!mbar_wait(p_full(s), gb[s] & 1, abort_flag, p.status)) { alive = false; break; }
            ++gb[s];
            tc_fence_after();
            const uint32_t o_tmem = tmem + 256 * s + 128;
#pragma unroll
            for (int k = 0; k < C::PV_KSTEPS; ++k) {
              const uint64_t bd =
                  smem_desc_sw128(sV + kv_off(s, t) + k * C::PV_KROWS * 128, C::KV_CHUNK, 1024);
              const uint32_t acc = (jj > 0 || k > 0) ? 1u : 0u;
              if (FP8)
                mma_fp8_ts(o_tmem, tmem + 256 * s + k * 8, bd, C::IDESC_PV, acc);
              else
                mma_bf16_ts(o_tmem, tmem + 256 * s + k * 8, bd, C::IDESC_PV, acc);
            }
            if constexpr (FP8 && PART == kFirstRow) {
              // diagonal block: the residual term P_lo (columns P_COLS.. of the slot)
#pragma unroll
              for (int k = 0; k < C::PV_KSTEPS; ++k) {
                const uint64_t bd =
                    smem_desc_sw128(sV + kv_off(s, t) + k * C::PV_KROWS * 128, C::KV_CHUNK, 1024);
                mma_fp8_ts(o_tmem, tmem + 256 * s + C::P_COLS + k * 8, bd, C::IDESC_PV, 1u);
              }
            }
            if (kEarlyK) {
              // S_{j+1} straight behind P V_j; the commits follow
              if (more) {
                issue_mmas_s(s, tk);
                mma_commit(s_full(s));
              }
              mma_commit(ve(s, t));
              if (!more) mma_commit(o_done(s));
            } else {
              // one-stage ring: release V_j's stage as soon as P V_j completes, so that
              // V_{j+1} loads while S_{j+1} runs
              mma_commit(ve(s, t));
              if (!more) mma_commit(o_done(s));
              if (more) {
                if (!mbar_wait(kf(s, tk), pk, abort_flag, p.status)) { alive = false; break; }
                tc_fence_after();
                issue_mmas_s(s, tk);
                mma_commit(s_full(s));
              }
            }
            ++itv[s];
            if (more) {
              mma_commit(ke(s, tk));
              if (jj + 2 == n) mma_commit(q_empty(s));  // the unit's last S: Q may be replaced
              ++itk[s];
            }
          }
        }
      }
      // drain: every tcgen05.mma issued by this thread has completed
      mma_commit(bar_drain);
      for (int spin = 0; spin < 4000000 && !mbar_try_wait(bar_drain, 0); ++spin) {}
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax + epilogue
    const int slot = (warp - 2) / 4;                 // which tile of the pair
    const int quad = warp % 4;                       // TMEM lane quadrant of this warp
    const int r = quad * 32 + lane;                  // query row within the tile
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t my_S = tmem + 256 * slot + lane_off;
    const uint32_t my_O = tmem + 256 * slot + 128 + lane_off;
    const float sl2 = p.scale_log2;
    uint32_t gb = 0, ot = 0;                         // blocks and units processed by this slot
    bool alive = true;
    for (int k = 0, u = blockIdx.x; u < p.total_units && alive; u = SNAKE ? snake_unit(p, ++k) : u + gridDim.x) {
      const Unit un = decode_unit<PART>(p, u);
      const int n = unit_len<DENSE>(p, un);
      if (n == 0 || (slot == 1 && !un.two)) continue;
      const int h = un.h0 + slot;
      // running max; sums of P that normalise O and, for the FP8 first row, of the
      // unrounded P (log-sum-exp)
      float m_run = -INFINITY;
      float2 l2 = make_float2(0.f, 0.f), lt2 = make_float2(0.f, 0.f);
      for (int jj = 0; jj < n; ++jj, ++gb) {
        if (!warp_wait(s_full(slot), gb & 1, abort_flag, p.status)) { alive = false; break; }
        tc_fence_after();
        uint32_t sr[BN];
#pragma unroll
        for (int c = 0; c < BN / 32; ++c) tmem_ld32(my_S + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[c * 32]));
        tmem_wait_ld();
        if (jj == n - 1) {
#pragma unroll
          for (int c = 0; c < BN; ++c)
            if (c > r) sr[c] = __float_as_uint(-INFINITY);
        }
        // row maximum with four independent chains
        float mq[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int c = 0; c < BN; c += 8)
#pragma unroll
          for (int q = 0; q < 4; ++q) mq[q] = max3f(mq[q], __uint_as_float(sr[c + 2 * q]), __uint_as_float(sr[c + 2 * q + 1]));
        const float mx = fmaxf(max3f(mq[0], mq[1], mq[2]), mq[3]);
        const float m_new = fmaxf(m_run, mx * sl2);
        const bool resc = m_new > m_run + 8.0f;
        const float m_use = resc ? m_new : m_run;
        const float alpha = resc ? ex2_approx(m_run - m_use) : 1.0f;
        const float m_sub = m_use == -INFINITY ? 0.f : m_use;
        const float2 sc2 = make_float2(sl2, sl2);
        const float2 bias2 = make_float2(p.p_bias - m_sub, p.p_bias - m_sub);
        float2 sq[4], tq4[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          sq[q] = make_float2(0.f, 0.f);
          tq4[q] = make_float2(0.f, 0.f);
        }
        // P is packed in place over the first P_COLS registers of sr (each pair or quad of
        // scores is read before its packed word is written).  FP8, diagonal block: P goes
        // to the product as two e4m3 terms, P = P_hi + P_lo with P_lo the rounded residual
        // of P_hi (stored after P_hi in TMEM and multiplied by V in a second product):
        // the diagonal block holds the first rows of a sequence, whose few keys would
        // otherwise carry e4m3's 2^-4 relative rounding straight into the output.
        auto exps = [&](auto want_lse) {
          if constexpr (!FP8) {
#pragma unroll
            for (int u2 = 0; u2 < BN / 2; ++u2) {
              const float2 y = fma2(make_float2(__uint_as_float(sr[2 * u2]), __uint_as_float(sr[2 * u2 + 1])), sc2, bias2);
              const uint32_t w = pack_bf16x2(ex2_approx(y.x), ex2_approx(y.y));
              sr[u2] = w;
              sq[u2 % 4] = add2(sq[u2 % 4], make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u)));
            }
          } else {
            // Rows 1..: O is normalised by the float32 sum of the unrounded weights (the
            // same sum the log-sum-exp takes).  First row (two-term P): by the sum of the
            // rounded terms, the e4m3 weights (exact in f16) going into two f16x2
            // accumulators, one weight per lane and quad (relative rounding 2^-11 per
            // addition), added in f32 every 16 quads.
            constexpr bool kRoundedSum = PART == kFirstRow;
            uint32_t hs[2] = {0u, 0u};
#pragma unroll
            for (int u4 = 0; u4 < BN / 4; ++u4) {
              const float2 y0 = fma2(make_float2(__uint_as_float(sr[4 * u4]), __uint_as_float(sr[4 * u4 + 1])), sc2, bias2);
              const float2 y1 = fma2(make_float2(__uint_as_float(sr[4 * u4 + 2]), __uint_as_float(sr[4 * u4 + 3])), sc2, bias2);
              const float2 e0 = make_float2(ex2_approx(y0.x), ex2_approx(y0.y));
              const float2 e1 = make_float2(ex2_approx(y1.x), ex2_approx(y1.y));
              const uint32_t w = __byte_perm(pack_e4m3x2(e0.x, e0.y), pack_e4m3x2(e1.x, e1.y), 0x5410);
              sr[u4] = w;
              if constexpr (!kRoundedSum) {
                sq[u4 % 4] = add2(sq[u4 % 4], add2(e0, e1));
              } else {
                uint32_t a, b;
                asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(a) : "h"(static_cast<uint16_t>(w & 0xFFFFu)));
                asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(b) : "h"(static_cast<uint16_t>(w >> 16)));
                hs[0] = hadd2_u32(hs[0], a);
                hs[1] = hadd2_u32(hs[1], b);
              }
              if (kRoundedSum && u4 % 16 == 15) {
                sq[(u4 / 16) % 4] = add2(sq[(u4 / 16) % 4], add2(h2_to_float2(hs[0]), h2_to_float2(hs[1])));
                hs[0] = 0u;
                hs[1] = 0u;
              }
              if constexpr (decltype(want_lse)::value) tq4[u4 % 4] = add2(tq4[u4 % 4], add2(e0, e1));
            }
          }
        };
        // LSEX (FP8 first row with a log-sum-exp requested): also the sums of the unrounded P
        exps(std::bool_constant<LSEX>{});
        if constexpr (FP8 && PART == kFirstRow) {
          {
            // residual pass (diagonal block only), before P_hi overwrites S in TMEM: S is
            // read again 32 columns at a time into score registers the pass above freed
            // (sr[64..95]); P_lo words go to sr[32..63] and then after P_hi in TMEM
#pragma unroll
            for (int c = 0; c < BN / 32; ++c) {
              tmem_ld32(my_S + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[64]));
              tmem_wait_ld();
#pragma unroll
              for (int q = 0; q < 8; ++q) {
                float x[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                  x[e] = __uint_as_float(sr[64 + 4 * q + e]);
                  if (c * 32 + 4 * q + e > r) x[e] = -INFINITY;
                }
                const float2 y0 = fma2(make_float2(x[0], x[1]), sc2, bias2);
                const float2 y1 = fma2(make_float2(x[2], x[3]), sc2, bias2);
                const uint32_t w = sr[8 * c + q];
                const float2 h01 = e4m3x2_to_float2(static_cast<uint16_t>(w & 0xFFFFu));
                const float2 h23 = e4m3x2_to_float2(static_cast<uint16_t>(w >> 16));
                const float2 r0 = make_float2(ex2_approx(y0.x) - h01.x, ex2_approx(y0.y) - h01.y);
                const float2 r1 = make_float2(ex2_approx(y1.x) - h23.x, ex2_approx(y1.y) - h23.y);
                const uint32_t wl = __byte_perm(pack_e4m3x2(r0.x, r0.y), pack_e4m3x2(r1.x, r1.y), 0x5410);
                sr[32 + 8 * c + q] = wl;
                sq[q % 4] = add2(sq[q % 4], e4m3x4_pairsum(wl));
              }
            }
            tmem_st32(my_S + C::P_COLS, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
          }
        }
        const float2 sum2 = add2(add2(sq[0], sq[1]), add2(sq[2], sq[3]));
        const float2 sumt2 = add2(add2(tq4[0], tq4[1]), add2(tq4[2], tq4[3]));
        static_assert(C::P_COLS % 32 == 0, "P columns");
#pragma unroll
        for (int c = 0; c < C::P_COLS / 32; ++c) tmem_st32(my_S + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[c * 32]));
        const float2 a2 = make_float2(alpha, alpha);
        l2 = fma2(l2, a2, sum2);
        if constexpr (LSEX) lt2 = fma2(lt2, a2, sumt2);
        if (jj > 0 && __any_sync(full, resc)) {
          // O holds the sum up to the previous block: S_j was issued after P V_{j-1},
          // the tensor core runs in order, and S_j is complete
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t o[32];
            tmem_ld32(my_O + c * 32, o);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; e += 2) {
              const float2 v = mul2(make_float2(__uint_as_float(o[e]), __uint_as_float(o[e + 1])), a2);
              o[e] = __float_as_uint(v.x);
              o[e + 1] = __float_as_uint(v.y);
            }
            tmem_st32(my_O + c * 32, o);
          }
        }
        tmem_wait_st();
        m_run = m_use;
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(p_full(slot));
      }
      if (!alive) break;
      // epilogue: wait for the unit's last P V product, normalise, store
      if (!warp_wait(o_done(slot), ot & 1, abort_flag, p.status)) { alive = false; break; }
      ++ot;
      tc_fence_after();
      const float l = l2.x + l2.y;
      const float inv = p.out_scale / l;
      const SeqInfo& sq = p.bt.seq[un.b];
      const int rows_valid = min(BN, sq.len - un.i * BN);
      const long long tok = static_cast<long long>(sq.tok0) + un.i * BN + r;
      unsigned char* orow = static_cast<unsigned char*>(p.out) + (tok * p.Hq + h) * D * 2;
      const float2 ii = make_float2(inv, inv);
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t o[32];
        tmem_ld32(my_O + c * 32, o);
        tmem_wait_ld();
        if (r < rows_valid) {
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint32_t w[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float2 v = mul2(make_float2(__uint_as_float(o[8 * q + 2 * e]), __uint_as_float(o[8 * q + 2 * e + 1])), ii);
              w[e] = pack_bf16x2(v.x, v.y);
            }
            *reinterpret_cast<uint4*>(orow + (c * 32 + 8 * q) * 2) = make_uint4(w[0], w[1], w[2], w[3]);
          }
        }
      }
      if (p.lse != nullptr && r < rows_valid) {
        // the sum of the unrounded weights (BF16: of the rounded ones; the factor is 1)
        const float lt = (LSEX ? lt2.x + lt2.y : l) / p.p_scale;
        p.lse[static_cast<long long>(h) * p.bt.total_tokens + tok] = (m_run + __log2f(lt)) * 0.69314718055994531f;
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

template <int D, int BN, bool FP8, bool PAGED, bool DENSE, int PART, bool SHKV, bool LSEX, bool SNAKE>
cudaError_t run_k(const BsaParams& prm, cudaStream_t st) {
  using C = Cfg<D, BN, FP8>;
  auto kern = bsa_kernel<D, BN, FP8, PAGED, DENSE, PART, SHKV, LSEX, SNAKE>;
  cudaError_t e = set_smem_once<bsa_kernel<D, BN, FP8, PAGED, DENSE, PART, SHKV, LSEX, SNAKE>>(C::SMEM_LAUNCH);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int grid = prm.total_units < sms ? prm.total_units : sms;
  if (grid <= 0) return cudaSuccess;
  kern<<<grid, kThreads, C::SMEM_LAUNCH, st>>>(prm);
  return cudaGetLastError();
}

// The FP8 first-row launch with a log-sum-exp requested keeps the unrounded P sums beside
// the rounded ones it normalises by (its own kernel, so the default one carries none of it)
template <int D, int BN, bool FP8, bool PAGED, bool DENSE, int PART, bool SHKV = false, bool SNAKE = false>
cudaError_t run(const BsaParams& prm, cudaStream_t st) {
  if constexpr (FP8 && PART == kFirstRow) {
    if (prm.lse != nullptr) return run_k<D, BN, FP8, PAGED, DENSE, PART, SHKV, true, SNAKE>(prm, st);
  }
  return run_k<D, BN, FP8, PAGED, DENSE, PART, SHKV, false, SNAKE>(prm, st);
}

template <int D, int BN, bool FP8, int PART>
cudaError_t run_part(const BsaParams& prm, bool paged, bool dense, cudaStream_t st) {
  // shared lists with an even group size: both heads of every pair walk one list of one
  // kv-head, so their K/V tiles are loaded once (instantiated for d = 128, block 128)
  if constexpr (D == 128 && BN == 128) {
    if (!dense && prm.list_group % 2 == 0)
      return paged ? run<D, BN, FP8, true, false, PART, true>(prm, st) : run<D, BN, FP8, false, false, PART, true>(prm, st);
  }
  if (paged)
    return dense ? run<D, BN, FP8, true, true, PART>(prm, st) : run<D, BN, FP8, true, false, PART>(prm, st);
  // an odd number of groups (e.g. a single head pair): the snake order (snake_unit); kept
  // out of the other kernels, whose round-robin loop it would otherwise slow
  if constexpr (PART != kFirstRow) {
    if (!dense && prm.groups % 2 == 1) return run<D, BN, FP8, false, false, PART, false, true>(prm, st);
  }
  return dense ? run<D, BN, FP8, false, true, PART>(prm, st) : run<D, BN, FP8, false, false, PART>(prm, st);
}

// BF16: one launch over all rows.  FP8: rows 1.. in the main launch, then each sequence's
// first q-block row (where rows have fewer keys than a block) in a small second launch.
template <int D, int BN, bool FP8>
cudaError_t run_mode(BsaParams prm, bool paged, bool dense, cudaStream_t st) {
  const int NP = (prm.Hq + 1) / 2;
  if constexpr (!FP8) {
    long long units = 0;
    for (int b = 0; b < prm.bt.num_seqs; ++b) units += static_cast<long long>(prm.bt.seq[b].nblk) * NP;
    prm.total_units = static_cast<int>(units);
    prm.groups = prm.bt.num_seqs * NP;
    return run_part<D, BN, FP8, kAllRows>(prm, paged, dense, st);
  } else {
    long long rest = 0;
    for (int b = 0; b < prm.bt.num_seqs; ++b) rest += static_cast<long long>(prm.bt.seq[b].nblk - 1) * NP;
    prm.total_units = static_cast<int>(rest);
    int busy = 0;  // sequences with rows after the first (ordered first)
    for (int b = 0; b < prm.bt.num_seqs; ++b) busy += prm.bt.seq[b].nblk > 1 ? 1 : 0;
    prm.groups = busy * NP;
    cudaError_t e = run_part<D, BN, FP8, kRestRows>(prm, paged, dense, st);
    if (e != cudaSuccess) return e;
    prm.total_units = prm.bt.num_seqs * NP;
    prm.groups = prm.bt.num_seqs * NP;
    prm.inject = 0;  // a test injection applies to the first launch only
    return run_part<D, BN, FP8, kFirstRow>(prm, paged, dense, st);
  }
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
  prm.list_group = a.list_group > 0 ? a.list_group : 1;
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
  // l is accumulated from the scaled P, so the V scale is all that remains
  prm.out_scale = fp8 ? a.v_scale : 1.0f;
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
