// Internal definitions shared by the libstem translation units: the batch
// description passed to every kernel by value, the device status word, and thin
// wrappers over the sm_100a PTX used by the kernels (mbarrier, TMA, tcgen05).
#pragma once

#include <cuda.h>
#include <atomic>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/stem.h"

namespace stem {

// ---------------------------------------------------------------- batch layout
struct SeqInfo {
  int tok0;            // first token of the sequence in the packed [T, H, d] tensors
  int len;             // tokens
  int nblk;            // N_b = ceil(len / B)
  int row0;            // first global block row (sum of N of earlier sequences)
  long long score0;    // offset of this sequence's packed causal scores within a head
  long long nnz0;      // offset of this sequence's selected pairs within a head
  long long nnz;       // K_b = sum_i k_i
  double r_start;      // TPD keep fraction of block row 0
};

struct Batch {
  int num_seqs;
  int total_rows;
  int total_tokens;
  int block;
  long long scores_per_head;
  long long nnz_per_head;
  double mu;
  SeqInfo seq[STEM_MAX_SEQS];
};

// Device status word bits (first 4 bytes of the workspace).
enum : uint32_t { kStatusTimeout = 1u, kStatusBounds = 2u };

// Workspace carve-up (all offsets 256-byte aligned).
struct WsLayout {
  size_t status;       // uint32 status word + debug words (256 B)
  size_t qbar;         // float [Hq, R, d]
  size_t kbar;         // float [Hkv, R, d]
  size_t lbar;         // float [Hkv, R]
  size_t scores;       // float [Hq, scores_per_head]
  size_t row_ptr;      // int32 [R + 1]
  size_t col_idx;      // int32 [Hq, nnz_per_head]
  size_t total;
};

// Raise a kernel's dynamic shared-memory limit once per device (the attribute outlives the
// call; setting it once also keeps the launch path free of non-stream calls, so a whole
// call can be captured into a CUDA graph).
template <auto KERN>
cudaError_t set_smem_once(int bytes) {
  static std::atomic<uint64_t> done{0};  // one bit per device ordinal (mod 64)
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = 1ull << (dev & 63);
  if (done.load(std::memory_order_acquire) & bit) return cudaSuccess;
  e = cudaFuncSetAttribute(KERN, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess) done.fetch_or(bit, std::memory_order_acq_rel);
  return e;
}

// ------------------------------------------------------------ device helpers
#if defined(__CUDACC__)

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_fence_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait: spins until the phase of the given parity has completed, or until
// `abort_flag` (shared) is raised by another warp, or until the time limit passes
// (then raises the abort flag and the device status word).  Returns true when the
// phase completed.
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s

__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          uint32_t* status) {
  if (mbar_try_wait(bar, parity)) return true;
  uint64_t t0 = global_ns();
  for (;;) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (global_ns() - t0 > kWaitLimitNs) {
      *abort_flag = 1;
      atomicOr(status, kStatusTimeout);
      return false;
    }
  }
}

// TMA: 3-D tiled load into shared memory, completion counted on an mbarrier.
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, uint32_t bar, int c0,
                                            int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

__device__ __forceinline__ void tma_prefetch_map(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ------------------------------------------------------------------ tcgen05
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// D[tmem] (+)= A[smem desc] * B[smem desc]; kind::f16 (bf16 inputs, fp32 accumulate)
__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// kind::f8f6f4 (e4m3 inputs, fp32 accumulate)
__device__ __forceinline__ void mma_fp8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                        uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive (once) on an mbarrier when all earlier tcgen05.mma of this thread completed.
__device__ __forceinline__ void mma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
               : "memory");
}

// 32 lanes x 32 columns of 32-bit TMEM -> 32 registers per thread.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
        "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
        "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
        "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]),
      "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]),
      "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
// D[tmem] (+)= A[tmem] * B[smem desc]: A (the M x K operand) read from tensor memory,
// one row per lane, K packed along 32-bit columns.
__device__ __forceinline__ void mma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void mma_fp8_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                           uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Packed fp32 pairs (sm_100): two lanes of arithmetic per instruction.
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
  unsigned long long ra, rb, rc, rd;
  asm("mov.b64 %0, {%1, %2};" : "=l"(ra) : "f"(a.x), "f"(a.y));
  asm("mov.b64 %0, {%1, %2};" : "=l"(rb) : "f"(b.x), "f"(b.y));
  asm("mov.b64 %0, {%1, %2};" : "=l"(rc) : "f"(c.x), "f"(c.y));
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(rd) : "l"(ra), "l"(rb), "l"(rc));
  float2 d;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(d.x), "=f"(d.y) : "l"(rd));
  return d;
}
__device__ __forceinline__ float2 add2(float2 a, float2 b) {
  unsigned long long ra, rb, rd;
  asm("mov.b64 %0, {%1, %2};" : "=l"(ra) : "f"(a.x), "f"(a.y));
  asm("mov.b64 %0, {%1, %2};" : "=l"(rb) : "f"(b.x), "f"(b.y));
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(rd) : "l"(ra), "l"(rb));
  float2 d;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(d.x), "=f"(d.y) : "l"(rd));
  return d;
}
__device__ __forceinline__ float2 mul2(float2 a, float2 b) {
  unsigned long long ra, rb, rd;
  asm("mov.b64 %0, {%1, %2};" : "=l"(ra) : "f"(a.x), "f"(a.y));
  asm("mov.b64 %0, {%1, %2};" : "=l"(rb) : "f"(b.x), "f"(b.y));
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(rd) : "l"(ra), "l"(rb));
  float2 d;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(d.x), "=f"(d.y) : "l"(rd));
  return d;
}
__device__ __forceinline__ float max3f(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// Shared-memory matrix descriptor, 128-byte swizzle (sm_100 version field = 1).
// lbo/sbo in bytes: K-major: sbo = byte stride between 8-row groups, lbo unused (16).
// MN-major: lbo = byte stride between 64-element (128 B) column chunks, sbo = byte
// stride between 8-row groups along K.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32;
  d |= static_cast<uint64_t>(1) << 46;
  d |= static_cast<uint64_t>(2) << 61;
  return d;
}

// Instruction descriptor: fp32 accumulator, A/B format codes (kind::f16: 1 = bf16;
// kind::f8f6f4: 0 = e4m3), majorness (0 = K-major, 1 = MN-major), M x N tile.
__host__ __device__ constexpr uint32_t instr_desc(uint32_t fmt, uint32_t a_mn_major, uint32_t b_mn_major,
                                                  uint32_t M, uint32_t N) {
  return (1u << 4) | (fmt << 7) | (fmt << 10) | (a_mn_major << 15) | (b_mn_major << 16) |
         ((N >> 3) << 17) | ((M >> 4) << 24);
}

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// Two floats -> two e4m3 codes in the low 16 bits (lo in bits 0..7), saturating.
__device__ __forceinline__ uint32_t pack_e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

// Two e4m3 codes (low byte first) -> two floats.
__device__ __forceinline__ float2 e4m3x2_to_float2(uint16_t v) {
  uint32_t h2;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(v));
  float lo, hi;
  asm("{\n\t.reg .f16 a, b;\n\tmov.b32 {a, b}, %2;\n\tcvt.f32.f16 %0, a;\n\tcvt.f32.f16 %1, b;\n\t}\n"
      : "=f"(lo), "=f"(hi)
      : "r"(h2));
  return make_float2(lo, hi);
}

// Packed f16 pair addition.
__device__ __forceinline__ uint32_t hadd2_u32(uint32_t a, uint32_t b) {
  uint32_t c;
  asm("add.rn.f16x2 %0, %1, %2;" : "=r"(c) : "r"(a), "r"(b));
  return c;
}

// An f16x2 word -> two floats (low half first).
__device__ __forceinline__ float2 h2_to_float2(uint32_t c) {
  float lo, hi;
  asm("{\n\t.reg .f16 x, y;\n\tmov.b32 {x, y}, %2;\n\tcvt.f32.f16 %0, x;\n\tcvt.f32.f16 %1, y;\n\t}\n"
      : "=f"(lo), "=f"(hi)
      : "r"(c));
  return make_float2(lo, hi);
}

// Four e4m3 codes (bytes 0..3) -> (b0 + b2, b1 + b3) as an f16x2 word: every e4m3 value is
// exact in f16, the pair sums are rounded to f16.
__device__ __forceinline__ uint32_t e4m3x4_pairsum_h(uint32_t v) {
  uint32_t a, b;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(a) : "h"(static_cast<uint16_t>(v & 0xFFFFu)));
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(b) : "h"(static_cast<uint16_t>(v >> 16)));
  return hadd2_u32(a, b);
}

// The same pair sums as floats.
__device__ __forceinline__ float2 e4m3x4_pairsum(uint32_t v) { return h2_to_float2(e4m3x4_pairsum_h(v)); }

// Locate the sequence owning a global block row.
__device__ __forceinline__ int seq_of_row(const Batch& bt, int row) {
  int b = 0;
  while (b + 1 < bt.num_seqs && bt.seq[b + 1].row0 <= row) ++b;
  return b;
}

// TPD budget of block row i (identical fp64 operation order on host and device;
// explicit round-to-nearest intrinsics keep the compiler from contracting).
__device__ __forceinline__ int tpd_k(double r, int N, double mu, int i) {
  double w;
  if (N == 1) {
    w = 1.0;
  } else {
    double t = __ddiv_rn(__dmul_rn(__dsub_rn(1.0, mu), static_cast<double>(i)), static_cast<double>(N - 1));
    w = __dmul_rn(__dsub_rn(1.0, t), static_cast<double>(i + 1));
  }
  double f = floor(__dmul_rn(r, w));
  int m = i + 1 < 2 ? i + 1 : 2;
  double kk = f < static_cast<double>(m) ? static_cast<double>(m) : f;
  if (kk > static_cast<double>(i + 1)) kk = static_cast<double>(i + 1);
  return static_cast<int>(kk);
}

#endif  // __CUDACC__

// Record a message for stem_last_error() and return the status (host).
stem_status_t set_last_error(stem_status_t s, const char* fmt, ...) __attribute__((format(printf, 2, 3)));

// ------------------------------------------------------------- host launchers
// One tensor of a pooling launch.
struct PoolTensor {
  const void* x;            // contiguous [T, H, d], or (paged) a cache [slots, P, H, d]
  int H;
  int paged;                // addressed through the block table
  float scale;              // FP8 dequant scale, 1 for bf16
  float* mean_out;          // [H, R, d] block means, or nullptr
  float* lognorm_out;       // [H, R] block means of log ||row||_2, or nullptr (exactly one of the two)
  int slices;               // set by the launcher: CTAs across a token row
};
// Q, K and V pooled in one launch (count tensors, in this order).
struct PoolSet {
  PoolTensor t[3];
  int count;
  const int32_t* block_table;  // paged tensors only
  int max_pages;
  int num_slots;            // slots of a paged cache
  uint32_t* status;         // device status word (a bad page slot sets the bounds bit)
};

cudaError_t launch_pool(const Batch& bt, const PoolSet& ps, int head_dim, bool fp8, cudaStream_t st);
cudaError_t launch_score(const Batch& bt, const float* qbar, const float* kbar, const float* lbar, int Hq, int Hkv,
                         int head_dim, float sigma, float beta, float* scores, cudaStream_t st);
// Scores computed inside the selection straight from the pooled summaries (no score
// matrix); the lists equal launch_score + launch_select's bit for bit.
bool fused_select_supported(int Hq, int Hkv, int group, int head_dim);
cudaError_t launch_select_fused(const Batch& bt, const float* qbar, const float* kbar, const float* lbar, int Hq,
                                int Hkv, int group, int head_dim, float sigma, float beta, int32_t* row_ptr,
                                int32_t* col_idx, uint32_t* status, cudaStream_t st);
// group = q-heads per list (1: a list per q-head; Hq/Hkv: a list per KV group)
cudaError_t launch_select(const Batch& bt, const float* scores, int Hq, int group, int32_t* row_ptr,
                          int32_t* col_idx, uint32_t* status, cudaStream_t st);

struct BsaArgs {
  const void* q;
  const void* k;            // contiguous K or paged k_cache
  const void* v;
  const int32_t* block_table;
  int max_pages;
  long long kv_rows;        // rows of the K/V tensor maps (T, or num_slots * page)
  const int32_t* row_ptr;   // nullptr in dense mode
  const int32_t* col_idx;
  int list_group;           // q-heads per list: 1, or Hq/Hkv with shared lists
  void* out;
  float* lse;
  int Hq, Hkv, head_dim;
  float sigma;
  float q_scale, k_scale, v_scale;
};

cudaError_t launch_bsa(const Batch& bt, const BsaArgs& a, bool fp8, bool paged, bool dense, uint32_t* status,
                       cudaStream_t st);

// Pending failure-injection request (stem_debug_inject); consumed by the next BSA launch.
int take_injection();
void set_injection(int mode);

}  // namespace stem
