// Shared device helpers: status word, mbarriers with bounded waits, TMA loads,
// tcgen05 (TMEM allocation, MMA, commit, loads) as inline PTX for sm_100a.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/moe_b200.h"

namespace moe {

// --------------------------------------------------------------------------
// Device status word (first 4 bytes of the workspace).
// --------------------------------------------------------------------------
__device__ __forceinline__ void set_status(int32_t* status, int32_t code) {
  if (status) atomicCAS(status, 0, code);
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// --------------------------------------------------------------------------
// mbarrier
// --------------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

// One bounded test of a phase.  The thread may sleep in it until the phase
// completes, for at most kSuspendNs: waiting warps then leave their issue slots
// to the warps that work (a GEMM's idle epilogue warps sleep through the main
// loop instead of polling beside the producer and MMA warps).
constexpr uint32_t kSuspendNs = 20000;
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(kSuspendNs)
      : "memory");
  return ok != 0;
}

// Wait until the phase with the given parity has completed.  Gives up after
// `limit_ns` of wall time or when *abort becomes non-zero; on a time-out it
// raises *abort and records MOE_ERR_TIMEOUT.  Returns true on success.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort,
                                          int32_t* status, uint64_t limit_ns = 2000000000ull) {
  if (mbar_try_wait(bar, parity)) return true;
  uint64_t t0 = global_timer_ns();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort) return false;
    if (global_timer_ns() - t0 > limit_ns) {
      *abort = 1;
      set_status(status, MOE_ERR_TIMEOUT);
      return false;
    }
  }
}

// Wait until the 32-bit counter at p reaches `target` (acquire, GPU scope),
// sleeping between polls; the same limit and abort handling as mbar_wait.
__device__ __forceinline__ bool counter_wait(const int32_t* p, int32_t target, volatile int* abort,
                                             int32_t* status, uint64_t limit_ns = 2000000000ull) {
  const uint64_t t0 = global_timer_ns();
  while (true) {
    int32_t v;
    asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    if (v >= target) return true;
    if (*abort) return false;
    if (global_timer_ns() - t0 > limit_ns) {
      *abort = 1;
      set_status(status, MOE_ERR_TIMEOUT);
      return false;
    }
    __nanosleep(200);
  }
}

// Orders this thread's earlier generic-proxy accesses (an acquire above) before
// its later async-proxy (TMA) accesses to global memory.
__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

// --------------------------------------------------------------------------
// TMA (no multicast anywhere in this library)
// --------------------------------------------------------------------------
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int32_t c0, int32_t c1, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      ".L2::cache_hint [%0], [%1, {%3, %4}], [%2], %5;" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "l"(policy)
      : "memory");
}

// 3-D tiled load; used for tile-major weights (one contiguous 16 KB tile per box).
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int32_t c0, int32_t c1, int32_t c2, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      ".L2::cache_hint [%0], [%1, {%3, %4, %5}], [%2], %6;" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2),
      "l"(policy)
      : "memory");
}

__device__ __forceinline__ uint64_t l2_policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

__device__ __forceinline__ uint64_t l2_policy_evict_last() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// --------------------------------------------------------------------------
// tcgen05
// --------------------------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}

__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T, kind::f16 (bf16 inputs, fp32 accumulate).
__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                         uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive on an mbarrier once all previously issued tcgen05 ops of this thread
// have completed.
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

// 32 lanes x 32 columns of 32-bit TMEM cells: thread i gets lane (base + i),
// columns c .. c+31 in r[0..31].
__device__ __forceinline__ void tmem_ld_32x32b_x32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
        "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
        "=r"(r[31])
      : "r"(taddr));
}

// As above with 16 columns: c .. c+15 in r[0..15].
__device__ __forceinline__ void tmem_ld_32x32b_x16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}

__device__ __forceinline__ void tmem_ld_wait() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Shared-memory matrix descriptor for a K-major tile written by TMA with
// 128-byte swizzling: rows of 128 bytes, 8-row groups 1024 bytes apart.
__device__ __forceinline__ uint64_t sdesc_kmajor_sw128(uint32_t saddr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4);  // start address
  d |= static_cast<uint64_t>(1) << 16;                   // leading byte offset (unused)
  d |= static_cast<uint64_t>(1024 >> 4) << 32;           // stride byte offset
  d |= static_cast<uint64_t>(1) << 46;                   // descriptor version (sm_100)
  d |= static_cast<uint64_t>(2) << 61;                   // 128-byte swizzle
  return d;
}

// Instruction descriptor, kind::f16 with bf16 A/B, fp32 D, both K-major.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N) {
  return (1u << 4)                                   // D format fp32
         | (1u << 7)                                 // A bf16
         | (1u << 10)                                // B bf16
         | (static_cast<uint32_t>(N >> 3) << 17)     // N / 8
         | (static_cast<uint32_t>(M >> 4) << 24);    // M / 16
}

__device__ __forceinline__ int lane_id() { return threadIdx.x & 31; }
__device__ __forceinline__ int warp_id() { return threadIdx.x >> 5; }

}  // namespace moe

namespace moe {

// 1-D bulk copy global -> shared, completing on an mbarrier (16-byte aligned,
// size a multiple of 16).
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes,
                                          uint64_t* bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint "
      "[%0], [%1], %2, [%3], %4;" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

// D[tmem] (+)= A * B^T with MXFP8 operands (e4m3) and e8m0 scales per 32 K
// elements read from TMEM; sf ids select the byte of the scale word.
__device__ __forceinline__ void mma_mxf8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                         uint32_t idesc, uint32_t sfa_tmem, uint32_t sfb_tmem,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}"
      ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem),
      "r"(sfb_tmem)
      : "memory");
}

// Copy one 128 x 4 scale-factor chunk (512 bytes: 32 rows of 16 bytes in
// shared memory) into TMEM lanes 0-127 (each 32-row group receives the same
// 32 x 128-bit block), 4 columns.
__device__ __forceinline__ void tmem_cp_sf_chunk(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc)
               : "memory");
}

// Descriptor of a contiguous 512-byte scale chunk: no swizzle, 8-row core
// matrices of 16-byte rows, 128 bytes apart.
__device__ __forceinline__ uint64_t sdesc_sf_chunk(uint32_t saddr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4);
  d |= static_cast<uint64_t>(128 >> 4) << 16;  // leading byte offset
  d |= static_cast<uint64_t>(128 >> 4) << 32;  // stride byte offset: next 8 rows
  d |= static_cast<uint64_t>(1) << 46;         // descriptor version (sm_100)
  return d;                                    // layout type 0: no swizzle
}

// Instruction descriptor, kind::mxf8f6f4 block-scaled: e4m3 A/B, e8m0 scales,
// both K-major, fp32 D; a_sf_id / b_sf_id pick the scale byte.
__device__ __forceinline__ uint32_t idesc_mxf8(int M, int N, uint32_t sf_id) {
  return (sf_id << 4)                                // b_sf_id
         | (0u << 7) | (0u << 10)                    // A, B: E4M3
         | (static_cast<uint32_t>(N >> 3) << 17)     // N / 8
         | (1u << 23)                                // scale format E8M0
         | (static_cast<uint32_t>(M >> 4) << 24)     // M / 16
         | (sf_id << 29);                            // a_sf_id
}

// Offset of block scale (row r, k-block kb) in the MMA scale layout of a
// matrix with KB k-blocks per row (KB % 4 == 0): 128-row x 4-block chunks of
// 512 bytes, chunk (r/128, kb/4) at index (r/128)*(KB/4) + kb/4, and inside a
// chunk byte (r%32)*16 + ((r%128)/32)*4 + kb%4.
__host__ __device__ __forceinline__ int64_t sf_offset(int64_t r, int kb, int KB) {
  return ((r >> 7) * (KB >> 2) + (kb >> 2)) * 512 + (r & 31) * 16 + ((r >> 5) & 3) * 4 + (kb & 3);
}

// MXFP8 scale code of a block from its amax (OCP MX rule: 2^(floor(log2 amax) - 8),
// biased exponent clamped to [0, 254]; amax 0 -> 127).
__device__ __forceinline__ uint32_t mx_scale_code(float amax) {
  if (amax == 0.0f) return 127u;
  const int e = static_cast<int>((__float_as_uint(amax) >> 23) & 0xFF);  // biased exponent
  const int code = e - 8;  // floor(log2 amax) - 8 + 127 for normal amax
  return static_cast<uint32_t>(code < 0 ? 0 : (code > 254 ? 254 : code));
}

// 2^(127 - code) as fp32 (code in [0, 253]), the exact reciprocal of the scale.
__device__ __forceinline__ float mx_inv_scale(uint32_t code) {
  return __uint_as_float((254u - code) << 23);
}

// fp32 -> e4m3 code, round to nearest even, saturating to +-448.
__device__ __forceinline__ uint8_t to_e4m3(float v) {
  uint16_t r;
  asm("{\n\t.reg .b16 t;\n\tcvt.rn.satfinite.e4m3x2.f32 t, %1, %2;\n\tmov.b16 %0, t;\n\t}"
      : "=h"(r)
      : "f"(0.0f), "f"(v));
  return static_cast<uint8_t>(r & 0xFF);
}

}  // namespace moe

namespace moe {

// D[tmem] (+)= A * B^T with NVFP4 operands (packed e2m1) and ue4m3 scales per
// 16 K elements read from TMEM (one 32-bit scale word per row per MMA).
__device__ __forceinline__ void mma_nvf4(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                         uint32_t idesc, uint32_t sfa_tmem, uint32_t sfb_tmem,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], "
      "p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
      : "memory");
}

// Instruction descriptor, kind::mxf4nvf4 block-scaled: e2m1 A/B, ue4m3 scales,
// K = 64 per MMA, both K-major, fp32 D.
__device__ __forceinline__ uint32_t idesc_nvf4(int M, int N) {
  return (1u << 7) | (1u << 10)                      // A, B: E2M1
         | (static_cast<uint32_t>(N >> 3) << 17)     // N / 8
         | (0u << 23)                                // scale format UE4M3
         | (static_cast<uint32_t>(M >> 4) << 24);    // M / 16
}

// Value of an e4m3 code (bias 7, 3 mantissa bits, subnormals at exponent 0);
// the codes used here are finite and non-negative.
__device__ __forceinline__ float e4m3_value(uint32_t c) {
  const uint32_t e = (c >> 3) & 15u, m = c & 7u;
  if (e == 0) return static_cast<float>(m) * 0.001953125f;  // m * 2^-9
  return __uint_as_float(((e + 120u) << 23) | (m << 20));    // (1 + m/8) * 2^(e-7)
}

// Two fp32 -> one byte of two e2m1 codes (round to nearest even, saturating
// at +-6); element `lo` in the low nibble, `hi` in the high nibble.
__device__ __forceinline__ uint32_t to_e2m1x2(float lo, float hi) {
  uint16_t r;
  asm("{\n\t.reg .b8 t;\n\tcvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\tcvt.u16.u8 %0, t;\n\t}"
      : "=h"(r)
      : "f"(hi), "f"(lo));
  return static_cast<uint32_t>(r) & 0xFFu;
}

// NVFP4 global encode scale 2688 / amax (448 * 6), 1 when amax is 0.
__device__ __forceinline__ float nv_global_scale(float amax) {
  return amax > 0.0f ? __fdiv_rn(2688.0f, amax) : 1.0f;
}

// Quantize 16 values of one NVFP4 block with global scale g.  Writes 8 bytes
// of packed codes and returns the ue4m3 block scale code.  Every step is one
// IEEE fp32 operation: t = (amax / 6) * g; sb = e4m3(t); r = g / value(sb);
// q = e2m1(v * r); a zero scale gives an all-zero block.
__device__ __forceinline__ uint32_t nv_quantize_block16(const float (&v)[16], float g,
                                                        uint32_t (&packed)[2]) {
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(v[i]));
  const float t = __fmul_rn(__fdiv_rn(amax, 6.0f), g);
  const uint32_t sb = to_e4m3(t) & 0x7Fu;
  if (sb == 0) {
    packed[0] = packed[1] = 0u;
    return 0u;
  }
  const float r = __fdiv_rn(g, e4m3_value(sb));
#pragma unroll
  for (int w = 0; w < 2; ++w) {
    uint32_t acc = 0;
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      const int i = w * 8 + 2 * b;
      acc |= to_e2m1x2(__fmul_rn(v[i], r), __fmul_rn(v[i + 1], r)) << (8 * b);
    }
    packed[w] = acc;
  }
  return sb;
}

// atomic max of a non-negative float stored as bits
__device__ __forceinline__ void atomic_max_nonneg(float* addr, float v) {
  atomicMax(reinterpret_cast<unsigned int*>(addr), __float_as_uint(v));
}

}  // namespace moe

namespace moe {

// Exclusive scan of ceil(counts[e] / P) * P over e < E into s_out[0..E]
// (E <= 1024), by a block of exactly 256 threads.
__device__ __forceinline__ void block_scan_padded(const int32_t* counts, int E, int P,
                                                  int32_t* s_out) {
  __shared__ int32_t warp_tot[8];
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  constexpr int PER = 4;
  int v[PER];
  int local = 0;
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const int e = tid * PER + i;
    const int c = e < E ? counts[e] : 0;
    v[i] = (c + P - 1) / P * P;
    local += v[i];
  }
  int incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int u = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += u;
  }
  if (lane == 31) warp_tot[w] = incl;
  __syncthreads();
  int run = incl - local;
  for (int i = 0; i < w; ++i) run += warp_tot[i];
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const int e = tid * PER + i;
    if (e <= E) s_out[e] = run;
    run += v[i];
  }
  if (tid == 255 && E == 4 * 256) s_out[E] = run;
  __syncthreads();
}

}  // namespace moe

namespace moe {

// Four rows of a 2-D tensor (row indices r0..r3, one 128-byte box row each)
// into consecutive shared-memory rows; out-of-range rows read as zeros.
__device__ __forceinline__ void tma_gather4(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int32_t c0, int32_t r0, int32_t r1, int32_t r2,
                                            int32_t r3, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile::gather4.mbarrier::complete_tx::bytes"
      ".L2::cache_hint [%0], [%1, {%3, %4, %5, %6, %7}], [%2], %8;" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(r0), "r"(r1),
      "r"(r2), "r"(r3), "l"(policy)
      : "memory");
}

}  // namespace moe

// --------------------------------------------------------------------------
// CTA pairs (cluster of two CTAs sharing one tcgen05 MMA, cta_group::2).
// Rank 0 of the pair issues the MMAs; each CTA holds half of the M rows of A
// and half of the N rows of B in its own shared memory and its own 128 TMEM
// lanes of the accumulator.  No multicast form of any instruction is used:
// completions that both CTAs must see are committed twice, once per CTA.
// --------------------------------------------------------------------------
namespace moe {

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// Address, in the cluster's shared window, of this CTA's `p` as seen in CTA `rank`.
__device__ __forceinline__ uint32_t cluster_addr(const void* p, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(p)), "r"(rank));
  return r;
}

__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;"
               ::: "memory");
}

// Arrive on an mbarrier given by its cluster address (possibly the peer's).
// Relaxed: the only user is the accumulator-empty signal, whose arriving
// threads have already waited for their TMEM loads (tcgen05.wait::ld) and
// hand no memory to the waiter.  A release at cluster scope first makes the
// thread's earlier memory operations visible cluster-wide, which measured
// 0.6-1.2 us per tile under a full HBM load, all of it stalling the next
// tile's MMAs.
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_bar) {
  asm volatile("mbarrier.arrive.relaxed.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_bar)
               : "memory");
}

// Arrive with release semantics at cluster scope (orders the thread's earlier
// reads and writes of either CTA's shared memory before the arrival).
__device__ __forceinline__ void mbar_arrive_release_cluster(uint32_t cluster_bar) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_bar)
               : "memory");
}

// mbar_wait with acquire semantics at cluster scope: pairs with arrivals made
// by the peer CTA (mbar_arrive_release_cluster), so the peer's earlier writes
// to this CTA's shared memory are visible afterwards.
__device__ __forceinline__ bool mbar_wait_cluster(uint64_t* bar, uint32_t parity,
                                                  volatile int* abort, int32_t* status,
                                                  uint64_t limit_ns = 2000000000ull) {
  const uint64_t t0 = global_timer_ns();
  while (true) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(kSuspendNs)
        : "memory");
    if (ok) return true;
    if (*abort) return false;
    if (global_timer_ns() - t0 > limit_ns) {
      *abort = 1;
      set_status(status, MOE_ERR_TIMEOUT);
      return false;
    }
  }
}

// 32-bit store to shared memory given by its cluster address (possibly the peer's).
__device__ __forceinline__ void st_shared_cluster_s32(uint32_t cluster_addr_, int32_t v) {
  asm volatile("st.shared::cluster.s32 [%0], %1;" ::"r"(cluster_addr_), "r"(v) : "memory");
}

__device__ __forceinline__ void tmem_alloc_pair(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}

__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}

// Tiled loads into this CTA's shared memory whose completion is counted on
// the mbarrier at `cluster_bar` (rank 0's barrier of the pair).
__device__ __forceinline__ void tma_load_2d_pair(void* dst, const CUtensorMap* map,
                                                 uint32_t cluster_bar, int32_t c0, int32_t c1,
                                                 uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      ".L2::cache_hint [%0], [%1, {%3, %4}], [%2], %5;" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(cluster_bar), "r"(c0), "r"(c1), "l"(policy)
      : "memory");
}

__device__ __forceinline__ void tma_load_3d_pair(void* dst, const CUtensorMap* map,
                                                 uint32_t cluster_bar, int32_t c0, int32_t c1,
                                                 int32_t c2, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      ".L2::cache_hint [%0], [%1, {%3, %4, %5}], [%2], %6;" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(cluster_bar), "r"(c0), "r"(c1), "r"(c2),
      "l"(policy)
      : "memory");
}

__device__ __forceinline__ void mma_bf16_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                              uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void mma_mxf8_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                              uint32_t idesc, uint32_t sfa_tmem,
                                              uint32_t sfb_tmem, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}"
      ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem),
      "r"(sfb_tmem)
      : "memory");
}

__device__ __forceinline__ void mma_nvf4_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                              uint32_t idesc, uint32_t sfa_tmem,
                                              uint32_t sfb_tmem, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], "
      "p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
      : "memory");
}

// Scale-factor chunk copy in both CTAs: each CTA's chunk at the same shared
// address goes to its own TMEM at taddr.
__device__ __forceinline__ void tmem_cp_sf_chunk_pair(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::2.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc)
               : "memory");
}

// Arrive on the mbarrier at `cluster_bar` once all prior tcgen05 ops of this
// thread (pair MMAs and copies) have completed.
__device__ __forceinline__ void mma_commit_pair(uint32_t cluster_bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          cluster_bar)
      : "memory");
}

}  // namespace moe

namespace moe {

// Programmatic dependent launch.  Every library kernel calls pdl_wait() before
// it reads or writes global memory: it returns once the preceding kernel in the
// stream has completed and its writes are visible (at once when the kernel was
// launched without the programmatic-serialization attribute).  pdl_trigger()
// lets the next kernel's CTAs start launching; they still wait in pdl_wait().
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

}  // namespace moe

namespace moe {

// One row copy by a warp: 16-byte vectors, the loads of eight vectors per lane
// issued before their stores (a zero source pointer writes zeros).  Plain
// loads on pointers that may alias the destination: the compiler cannot sink
// them to their stores, so the eight stay in flight together.
__device__ __forceinline__ void warp_copy_row(uint4* d, const uint4* s, int vecs, int lane) {
  for (int v0 = 0; v0 < vecs; v0 += 32 * 8) {
    uint4 buf[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int v = v0 + i * 32 + lane;
      buf[i] = (s && v < vecs) ? s[v] : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int v = v0 + i * 32 + lane;
      if (v < vecs) d[v] = buf[i];
    }
  }
}

}  // namespace moe
