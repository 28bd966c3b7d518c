// Block-sparse causal flash-attention prefill on sm_100a (tcgen05 + TMEM + TMA).
//
// Tencent Cloud article "从Stem稀疏注意力看 大模型推理的架构取舍", section
// "HPC-BSA：跳块零开销的秘密": for each Q block the kernel holds the list of KV
// blocks to visit and its inner loop walks only that list, with no per-block
// "skip?" branch; a skipped block is mathematically the same as all its scores
// being -inf, so the softmax stays exact; the inner path is the dense one.  The
// same section notes native support for a paged KV cache.
//
// Design (one CTA per SM, persistent over (q-head, q-block) tiles, 6 warps):
//   warp 0      TMA producer: Q tile once per tile, then K_j, V_j for every listed j
//               into a 2-stage ring (64-row boxes, 128-byte swizzle; a paged cache
//               is addressed page by page through the block table).
//   warp 1      MMA issuer (one thread): S = Q K_j^T into one of two TMEM S buffers,
//               then O += P_j V_j into the TMEM O accumulator.  S_{j+1} is issued
//               before P_j is ready so the tensor core overlaps the softmax.
//   warps 2..5  softmax (one thread per query row, TMEM lane quadrant = warp % 4):
//               online softmax in the log2 domain, token-level causal mask on the
//               diagonal block only (always the last list entry), lazy rescaling
//               of O (only when the running max grows by more than 2^8), P written
//               to shared memory for the P V product, then the epilogue (O / l ->
//               bf16, log-sum-exp).
// Every mbarrier wait is bounded (2 s); on expiry the CTA raises an abort flag,
// records STEM_ERR_TIMEOUT in the status word, drains its tensor-core work and
// releases its TMEM before exiting.
#include <string.h>

#include "stem_internal.cuh"

namespace stem {
namespace {

constexpr int kBM = 128;         // query rows per tile (tcgen05 M)
constexpr int kStages = 2;       // K/V ring depth
constexpr int kThreads = 192;    // 6 warps
constexpr uint32_t kTmemCols = 512;

template <int D, int BN, bool FP8>
struct Cfg {
  static constexpr int ES = FP8 ? 1 : 2;
  static constexpr int CH = 128 / ES;             // elements per 128-byte swizzle row
  static constexpr int DCH = D * ES / 128;        // 128-byte chunks along d
  static constexpr int PCH = BN * ES / 128;       // 128-byte chunks along a P row
  static_assert(D * ES % 128 == 0 && BN * ES % 128 == 0, "rows must be whole 128-byte swizzle rows");
  static constexpr int Q_CHUNK = kBM * 128;
  static constexpr int KV_CHUNK = BN * 128;
  static constexpr int Q_BYTES = kBM * D * ES;
  static constexpr int KV_BYTES = BN * D * ES;
  static constexpr int P_BYTES = kBM * BN * ES;
  static constexpr int S_KSTEPS = D * ES / 32;    // MMAs along d for S (32 bytes of K each)
  static constexpr int PV_KSTEPS = BN * ES / 32;  // MMAs along the KV block for O
  static constexpr int PV_KROWS = 32 / ES;        // KV rows consumed per PV MMA
  static constexpr int HALVES = BN / 64;          // 64-row TMA boxes per KV block
  // shared memory carve-up (all tiles 1024-byte aligned for the 128-byte swizzle)
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + Q_BYTES;
  static constexpr int OFF_V = OFF_K + kStages * KV_BYTES;
  static constexpr int OFF_P = OFF_V + kStages * KV_BYTES;
  static constexpr int OFF_BAR = OFF_P + 2 * P_BYTES;
  static constexpr int SMEM = OFF_BAR + 256 + 1024;  // + barriers + alignment slack
  // force one CTA per SM (TMEM allocation takes all 512 columns)
  static constexpr int SMEM_LAUNCH = SMEM < 120 * 1024 ? 120 * 1024 : SMEM;
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
  float out_scale;   // FP8: v_scale (l carries p_scale); BF16: 1
  float p_scale;     // FP8: P is multiplied by this before rounding to e4m3
  uint32_t* status;
  signed char order[STEM_MAX_SEQS];  // sequences by decreasing block count
};

struct Tile {
  int b, i, h;
};

__device__ __forceinline__ Tile decode_tile(const BsaParams& p, int t) {
  Tile r{0, 0, 0};
  int acc = 0;
  for (int q = 0; q < p.bt.num_seqs; ++q) {
    const int b = p.order[q];
    const int nt = p.bt.seq[b].nblk * p.Hq;
    if (t < acc + nt) {
      const int local = t - acc;
      r.b = b;
      r.i = p.bt.seq[b].nblk - 1 - local / p.Hq;
      r.h = local % p.Hq;
      return r;
    }
    acc += nt;
  }
  return r;
}

// Warp-uniform bounded wait on an mbarrier phase (see stem_internal.cuh).
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          uint32_t* status) {
  const unsigned full = 0xffffffffu;
  int spins = 0;
  uint64_t t0 = 0;
  for (;;) {
    const bool ok = mbar_try_wait(bar, parity);
    if (__all_sync(full, ok)) return true;
    const int ab = __shfl_sync(full, *abort_flag, 0);
    if (ab) return false;
    if (++spins == 8) t0 = global_ns();
    if (spins > 8) {
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
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t sQ = sbase + C::OFF_Q;
  const uint32_t sK = sbase + C::OFF_K;
  const uint32_t sV = sbase + C::OFF_V;
  const uint32_t sP = sbase + C::OFF_P;
  unsigned char* bar_area = smem + C::OFF_BAR;
  // barriers (8 bytes each)
  const uint32_t b0 = sbase + C::OFF_BAR;
  const uint32_t bar_q_full = b0 + 0, bar_q_empty = b0 + 8;
  const uint32_t bar_k_full = b0 + 16, bar_k_empty = b0 + 32;   // [2]
  const uint32_t bar_v_full = b0 + 48, bar_v_empty = b0 + 64;   // [2]
  const uint32_t bar_s_full = b0 + 80, bar_s_empty = b0 + 96;   // [2]
  const uint32_t bar_p_full = b0 + 112, bar_pv_done = b0 + 120;
  const uint32_t bar_drain = b0 + 128;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_area + 160);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bar_area + 168);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  if (threadIdx.x == 0) {
    mbar_init(bar_q_full, 1);
    mbar_init(bar_q_empty, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bar_k_full + 8 * s, 1);
      mbar_init(bar_k_empty + 8 * s, 1);
      mbar_init(bar_v_full + 8 * s, 1);
      mbar_init(bar_v_empty + 8 * s, 1);
      mbar_init(bar_s_full + 8 * s, 1);
      mbar_init(bar_s_empty + 8 * s, 4);
    }
    mbar_init(bar_p_full, 4);
    mbar_init(bar_pv_done, 1);
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
  const uint32_t tmem_S = tmem;          // two buffers at columns 0 and 128
  const uint32_t tmem_O = tmem + 256;    // D columns

  const int G = p.Hq / p.Hkv;
  const unsigned full = 0xffffffffu;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_map(&p.tq);
      tma_prefetch_map(&p.tk);
      tma_prefetch_map(&p.tv);
    }
    uint32_t it = 0, tq = 0;
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
        int jl = j0 + lane;
        int myj = jl;
        if (!DENSE) myj = jl < n ? __ldg(list + jl) : 0;
        if (jl < n && (myj < 0 || myj > tl.i)) {
          atomicOr(p.status, kStatusBounds);
          myj = tl.i;
        }
        if (jl >= n) myj = 0;
        // rows of this lane's block (one per 64-row half), resolved through the block table
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
          const uint32_t st = it % kStages, ph = (it / kStages) & 1;
          if (!warp_wait(bar_k_empty + 8 * st, ph ^ 1, abort_flag, p.status)) { alive = false; break; }
          if (lane == 0) {
            mbar_arrive_expect_tx(bar_k_full + 8 * st, C::KV_BYTES);
            for (int c = 0; c < C::DCH; ++c)
              for (int hh = 0; hh < C::HALVES; ++hh)
                tma_load_3d(sK + st * C::KV_BYTES + c * C::KV_CHUNK + hh * 64 * 128, &p.tk, bar_k_full + 8 * st,
                            c * C::CH, kvh, rows[hh]);
          }
          if (!warp_wait(bar_v_empty + 8 * st, ph ^ 1, abort_flag, p.status)) { alive = false; break; }
          if (lane == 0) {
            mbar_arrive_expect_tx(bar_v_full + 8 * st, C::KV_BYTES);
            for (int c = 0; c < C::DCH; ++c)
              for (int hh = 0; hh < C::HALVES; ++hh)
                tma_load_3d(sV + st * C::KV_BYTES + c * C::KV_CHUNK + hh * 64 * 128, &p.tv, bar_v_full + 8 * st,
                            c * C::CH, kvh, rows[hh]);
          }
          ++it;
        }
      }
    }
    if (!alive) {
      // let the copies already issued land before the CTA can exit
      for (uint32_t q = (it > kStages ? it - kStages : 0); q < it; ++q) {
        const uint32_t st = q % kStages, ph = (q / kStages) & 1;
        for (int spin = 0; spin < 1000000 && !mbar_try_wait(bar_k_full + 8 * st, ph); ++spin) {}
        for (int spin = 0; spin < 1000000 && !mbar_try_wait(bar_v_full + 8 * st, ph); ++spin) {}
      }
      if (tq > 0)
        for (int spin = 0; spin < 1000000 && !mbar_try_wait(bar_q_full, (tq - 1) & 1); ++spin) {}
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    uint32_t it_s = 0, it_v = 0, is = 0, ip = 0, tq = 0;
    bool alive = true;
    auto issue_s = [&](void) -> bool {
      const uint32_t sb = is % 2, sph = (is / 2) & 1;
      const uint32_t st = it_s % kStages, kph = (it_s / kStages) & 1;
      if (!warp_wait(bar_s_empty + 8 * sb, sph ^ 1, abort_flag, p.status)) return false;
      if (!warp_wait(bar_k_full + 8 * st, kph, abort_flag, p.status)) return false;
      tc_fence_after();
      if (lane == 0) {
#pragma unroll
        for (int ks = 0; ks < C::S_KSTEPS; ++ks) {
          const int c = ks / 4, w = ks % 4;
          const uint64_t ad = smem_desc_sw128(sQ + c * C::Q_CHUNK + w * 32, 16, 1024);
          const uint64_t bd = smem_desc_sw128(sK + st * C::KV_BYTES + c * C::KV_CHUNK + w * 32, 16, 1024);
          if (FP8)
            mma_fp8(tmem_S + sb * 128, ad, bd, C::IDESC_S, ks > 0);
          else
            mma_bf16(tmem_S + sb * 128, ad, bd, C::IDESC_S, ks > 0);
        }
        mma_commit(bar_s_full + 8 * sb);
        mma_commit(bar_k_empty + 8 * st);
      }
      __syncwarp();
      ++is;
      ++it_s;
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
        const uint32_t st = it_v % kStages, vph = (it_v / kStages) & 1;
        if (!warp_wait(bar_v_full + 8 * st, vph, abort_flag, p.status)) { alive = false; break; }
        tc_fence_after();
        if (lane == 0) {
#pragma unroll
          for (int ks = 0; ks < C::PV_KSTEPS; ++ks) {
            const int c = (ks * 32) / 128, w = ks % 4;
            const uint64_t ad = smem_desc_sw128(sP + pb * C::P_BYTES + c * C::Q_CHUNK + w * 32, 16, 1024);
            const uint64_t bd = smem_desc_sw128(sV + st * C::KV_BYTES + ks * C::PV_KROWS * 128, C::KV_CHUNK, 1024);
            if (FP8)
              mma_fp8(tmem_O, ad, bd, C::IDESC_PV, (jj > 0 || ks > 0) ? 1u : 0u);
            else
              mma_bf16(tmem_O, ad, bd, C::IDESC_PV, (jj > 0 || ks > 0) ? 1u : 0u);
          }
          mma_commit(bar_v_empty + 8 * st);
          mma_commit(bar_pv_done);
        }
        __syncwarp();
        ++it_v;
      }
    }
    // drain: every tcgen05.mma issued by this thread has completed
    if (lane == 0) mma_commit(bar_drain);
    __syncwarp();
    for (int spin = 0; spin < 4000000 && !mbar_try_wait(bar_drain, 0); ++spin) {}
  } else {
    // ------------------------------------------------------------ softmax + epilogue
    const int quad = warp % 4;
    const int r = quad * 32 + lane;                  // query row within the tile
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    uint32_t is = 0, ipv = 0, ipw = 0;
    bool alive = true;
    for (int t = blockIdx.x; t < p.total_tiles && alive; t += gridDim.x) {
      const Tile tl = decode_tile(p, t);
      const int32_t* list;
      const int n = tile_len<DENSE>(p, tl, &list);
      if (n == 0) continue;
      // l_run: sum of the rounded P the P.V product sees (normalises O);
      // lt_run (FP8 only): sum of the unrounded P (gives the log-sum-exp)
      float m_run = -INFINITY, l_run = 0.f, lt_run = 0.f;
      for (int jj = 0; jj < n; ++jj) {
        const uint32_t sb = is % 2, sph = (is / 2) & 1;
        if (!warp_wait(bar_s_full + 8 * sb, sph, abort_flag, p.status)) { alive = false; break; }
        ++is;
        tc_fence_after();
        uint32_t sr[BN];
#pragma unroll
        for (int c = 0; c < BN / 32; ++c) tmem_ld32(tmem_S + sb * 128 + lane_off + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[c * 32]));
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_s_empty + 8 * sb);
        const bool diag = (jj == n - 1);
        float mx = -INFINITY;
#pragma unroll
        for (int c = 0; c < BN; ++c) {
          float v = __uint_as_float(sr[c]);
          if (diag && c > r) v = -INFINITY;
          sr[c] = __float_as_uint(v);
          mx = fmaxf(mx, v);
        }
        const float m_new = fmaxf(m_run, mx * p.scale_log2);
        const bool resc = m_new > m_run + 8.0f;
        const float m_use = resc ? m_new : m_run;
        const float alpha = resc ? ex2_approx(m_run - m_use) : 1.0f;
        // P = exp2(s * scale - m), written to the P buffer of this block (swizzled)
        const uint32_t pbuf = sP + (ipw % 2) * C::P_BYTES;
        ++ipw;
        float sum = 0.f, sum_t = 0.f;
        if (!FP8) {
#pragma unroll
          for (int u = 0; u < BN / 8; ++u) {
            uint32_t w4[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float p0 = ex2_approx(fmaf(__uint_as_float(sr[8 * u + 2 * e]), p.scale_log2, -m_use));
              const float p1 = ex2_approx(fmaf(__uint_as_float(sr[8 * u + 2 * e + 1]), p.scale_log2, -m_use));
              w4[e] = pack_bf16x2(p0, p1);
              // normalise with the rounded weights the P.V product uses
              sum += __uint_as_float(w4[e] << 16) + __uint_as_float(w4[e] & 0xFFFF0000u);
            }
            const int chunk = u / 8, uu = u % 8;
            const uint32_t addr = pbuf + chunk * C::Q_CHUNK + r * 128 + ((uu ^ (r & 7)) << 4);
            asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(w4[0]), "r"(w4[1]), "r"(w4[2]),
                         "r"(w4[3])
                         : "memory");
          }
        } else {
#pragma unroll
          for (int u = 0; u < BN / 16; ++u) {
            uint32_t w4[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              float pv[4];
#pragma unroll
              for (int q = 0; q < 4; ++q)
                pv[q] = ex2_approx(fmaf(__uint_as_float(sr[16 * u + 4 * e + q]), p.scale_log2, -m_use));
              sum_t += (pv[0] + pv[1]) + (pv[2] + pv[3]);
              const uint32_t lo = pack_e4m3x2(pv[0] * p.p_scale, pv[1] * p.p_scale);
              const uint32_t hi = pack_e4m3x2(pv[2] * p.p_scale, pv[3] * p.p_scale);
              w4[e] = lo | (hi << 16);
              // normalise with the rounded (scaled) weights the P.V product uses
              const float2 a = e4m3x2_to_float2(static_cast<uint16_t>(lo));
              const float2 b = e4m3x2_to_float2(static_cast<uint16_t>(hi));
              sum += (a.x + a.y) + (b.x + b.y);
            }
            const uint32_t addr = pbuf + r * 128 + ((u ^ (r & 7)) << 4);
            asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(w4[0]), "r"(w4[1]), "r"(w4[2]),
                         "r"(w4[3])
                         : "memory");
          }
        }
        l_run = l_run * alpha + sum;
        if (FP8) lt_run = lt_run * alpha + sum_t;
        fence_proxy_async_smem();
        if (jj > 0) {
          // O holds the sum up to block jj-1 once its P V product is done
          if (!warp_wait(bar_pv_done, ipv & 1, abort_flag, p.status)) { alive = false; break; }
          ++ipv;
          tc_fence_after();
          if (__any_sync(full, resc)) {
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
              uint32_t o[32];
              tmem_ld32(tmem_O + lane_off + c * 32, o);
              tmem_wait_ld();
#pragma unroll
              for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
              tmem_st32(tmem_O + lane_off + c * 32, o);
            }
            tmem_wait_st();
          }
        }
        m_run = m_use;
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_p_full);
      }
      if (!alive) break;
      // epilogue: wait for the last P V product, normalise, store
      if (!warp_wait(bar_pv_done, ipv & 1, abort_flag, p.status)) { alive = false; break; }
      ++ipv;
      tc_fence_after();
      const SeqInfo& s = p.bt.seq[tl.b];
      const int rows_valid = min(BN, s.len - tl.i * BN);
      const float inv = p.out_scale / l_run;
      const long long tok = static_cast<long long>(s.tok0) + tl.i * BN + r;
      unsigned char* orow = static_cast<unsigned char*>(p.out) + (tok * p.Hq + tl.h) * D * 2;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t o[32];
        tmem_ld32(tmem_O + lane_off + c * 32, o);
        tmem_wait_ld();
        if (r < rows_valid) {
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint4 v;
            v.x = pack_bf16x2(__uint_as_float(o[8 * q + 0]) * inv, __uint_as_float(o[8 * q + 1]) * inv);
            v.y = pack_bf16x2(__uint_as_float(o[8 * q + 2]) * inv, __uint_as_float(o[8 * q + 3]) * inv);
            v.z = pack_bf16x2(__uint_as_float(o[8 * q + 4]) * inv, __uint_as_float(o[8 * q + 5]) * inv);
            v.w = pack_bf16x2(__uint_as_float(o[8 * q + 6]) * inv, __uint_as_float(o[8 * q + 7]) * inv);
            *reinterpret_cast<uint4*>(orow + (c * 32 + 8 * q) * 2) = v;
          }
        }
      }
      if (p.lse != nullptr && r < rows_valid)
        p.lse[static_cast<long long>(tl.h) * p.bt.total_tokens + tok] =
            (m_run + __log2f(FP8 ? lt_run : l_run)) * 0.69314718055994531f;
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
  const float log2e = 1.4426950408889634f;
  prm.scale_log2 = a.sigma * (fp8 ? a.q_scale * a.k_scale : 1.0f) * log2e;
  // FP8: P <= 2^8 after the lazy max update; 448 / 256 keeps it inside e4m3's range.
  prm.p_scale = fp8 ? 1.75f : 1.0f;
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
