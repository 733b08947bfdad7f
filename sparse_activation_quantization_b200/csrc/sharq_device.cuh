// sharq_device.cuh - device helpers shared by the SharQ kernels (sm_100a).
//
// Three groups:
//   1. NVFP4 scalar arithmetic (E2M1 / E4M3 conversion and decode) written
//      from the format definitions; conversions to the 4- and 8-bit formats
//      use the hardware cvt.rn.satfinite instructions.
//   2. The tiled operand layouts of include/sharq.h (byte offsets).
//   3. Thin inline-PTX wrappers: mbarrier, bulk copy (TMA engine), and the
//      tcgen05 family (TMEM alloc, smem->TMEM copy, block-scaled MMA, loads).
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace sharq {

constexpr int kTileRows = 128;
constexpr int kTileK = 256;
// tile sizes in bytes (see include/sharq.h)
constexpr int kCodesTile = 16384;   // 128 rows x 128 B, 128-byte swizzle
constexpr int kSpTile = 8192;       // 128 rows x 64 B, 64-byte swizzle
constexpr int kMetaTile = 2048;     // 128 rows x 16 B
constexpr int kSf32Tile = 1024;     // 2 scale atoms
constexpr int kSf64Tile = 512;      // 1 scale atom (MXFP4 backbone: one scale per 64 logical K)
constexpr int kSf16Tile = 2048;     // 4 scale atoms
constexpr float kGlobalDiv = 2688.0f;  // 6 (E2M1 max) * 448 (E4M3 max)

// ------------------------------------------------------------ formats ----

// two floats -> one byte of E2M1 codes, `lo` in the low nibble
__device__ __forceinline__ uint32_t cvt_e2m1x2(float lo, float hi) {
  uint32_t out;
  asm("{\n\t.reg .b8 q;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 q, %1, %2;\n\t"
      "cvt.u32.u8 %0, q;\n\t}"
      : "=r"(out) : "f"(hi), "f"(lo));
  return out & 0xFFu;
}

// non-negative float -> E4M3 byte (round to nearest even, saturate to 448)
__device__ __forceinline__ uint32_t cvt_e4m3(float x) {
  uint32_t out;
  asm("{\n\t.reg .b16 q;\n\t"
      "cvt.rn.satfinite.e4m3x2.f32 q, %1, %2;\n\t"
      "cvt.u32.u16 %0, q;\n\t}"
      : "=r"(out) : "f"(0.0f), "f"(x));
  return out & 0xFFu;
}

// E4M3 byte (sign bit clear) -> float, exact.  Definition: exponent field e
// (bias 7), mantissa m: e == 0 -> m * 2^-9, else (8 + m) * 2^(e - 10).
__device__ __forceinline__ float e4m3_value(uint32_t b) {
  uint32_t e = (b >> 3) & 15u, m = b & 7u;
  if (e == 0) return __fmul_rn((float)m, 0x1p-9f);
  return __uint_as_float(((e + 120u) << 23) | (m << 20));
}

// E2M1 code -> float, exact.  Twice the magnitudes {0,.5,1,1.5,2,3,4,6} are
// the nibbles of 0xC8643210.
__device__ __forceinline__ float e2m1_value(uint32_t c) {
  float mag = __fmul_rn((float)((0xC8643210u >> (4u * (c & 7u))) & 0xFu), 0.5f);
  return (c & 8u) ? -mag : mag;
}

// One NVFP4 block scale: sb = E4M3(f32(amax / f32(6*s))), S = f32(dec*s),
// inv = S > 0 ? f32(1/S) : 0.
struct BlockScale {
  uint32_t sb;
  float dec;
  float inv;
};

__device__ __forceinline__ BlockScale block_scale(float amax, float six_s, float s) {
  BlockScale r;
  r.sb = cvt_e4m3(__fdiv_rn(amax, six_s));
  r.dec = e4m3_value(r.sb);
  float S = __fmul_rn(r.dec, s);
  r.inv = S > 0.0f ? __frcp_rn(S) : 0.0f;
  return r;
}

// MX block scale (OCP Microscaling Formats v1.0, E8M0): X = 2^e with
// e = floor(log2 amax) - 2 (E2M1's largest exponent), clamped to [-127, 127];
// -127 for an all-zero block.  floor(log2) is read off the float32 encoding.
__device__ __forceinline__ float pow2f(int e) {  // exact 2^e for e in [-127, 127]
  return e >= -126 ? __uint_as_float((uint32_t)(e + 127) << 23) : __uint_as_float(0x00400000u);
}
__device__ __forceinline__ BlockScale mx_block_scale(float amax) {
  const uint32_t ef = __float_as_uint(amax) >> 23;  // amax >= 0
  int e = ef > 0 ? (int)ef - 127 - 2 : -127;       // zero and subnormal blocks clamp to -127
  e = e < -127 ? -127 : (e > 127 ? 127 : e);
  BlockScale r;
  r.sb = (uint32_t)(e + 127);
  r.dec = pow2f(e);
  r.inv = pow2f(-e);
  return r;
}

// ------------------------------------------------------------ layouts ----

// byte offset, within a 16 KB codes tile, of 16-byte chunk q (0..7) of row r
__device__ __host__ __forceinline__ uint32_t codes_chunk_off(uint32_t r, uint32_t q) {
  return r * 128u + ((q ^ (r & 7u)) << 4);
}
// byte offset, within an 8 KB sparse-codes tile, of 16-byte chunk q (0..3)
__device__ __host__ __forceinline__ uint32_t sp_chunk_off(uint32_t r, uint32_t q) {
  return r * 64u + ((q ^ ((r >> 1) & 3u)) << 4);
}
// byte offset of scale i (0..3) of atom a for row r inside a scale tile
__device__ __host__ __forceinline__ uint32_t sf_off(uint32_t r, uint32_t atom, uint32_t i) {
  return atom * 512u + (r & 31u) * 16u + (r >> 5) * 4u + i;
}

// ------------------------------------------------------------ PTX: misc --

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ------------------------------------------------------------ mbarrier ---

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait for the phase of parity `parity` to complete.  Returns false
// once the global timer passes `deadline` or *abort becomes non-zero.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, uint64_t deadline,
                                          volatile int* abort) {
  while (!mbar_try_wait(bar, parity)) {
    if (*abort) return false;
    if (globaltimer_ns() > deadline) return false;
  }
  return true;
}

// ------------------------------------------------------------ clusters ---

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// all threads of all CTAs of the cluster (used once, right after start-up)
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// shared::cta address -> the same offset in CTA `rank` of this cluster
__device__ __forceinline__ uint32_t mapa_shared(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}
// arrive (release, cluster scope) on an mbarrier of another CTA
__device__ __forceinline__ void mbar_arrive_remote(uint32_t remote_bar) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(remote_bar) : "memory");
}
// relaxed arrive on an mbarrier of another CTA: orders none of this thread's
// earlier memory operations (a release at cluster scope costs ~0.7 us on
// B200).  For signals whose data is not written by this thread: TMA bytes
// that already completed this CTA's own barrier, or TMEM loads already waited
// for with tcgen05.wait::ld.
__device__ __forceinline__ void mbar_arrive_remote_relaxed(uint32_t remote_bar) {
  asm volatile("mbarrier.arrive.relaxed.cluster.shared::cluster.b64 _, [%0];" ::"r"(remote_bar) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait_cluster(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait with cluster-scope acquire, for barriers that peers arrive on
__device__ __forceinline__ bool mbar_wait_cluster(uint64_t* bar, uint32_t parity, uint64_t deadline,
                                                  volatile int* abort) {
  while (!mbar_try_wait_cluster(bar, parity)) {
    if (*abort) return false;
    if (globaltimer_ns() > deadline) return false;
  }
  return true;
}
__device__ __forceinline__ float4 ld_shared_cluster_f4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(addr)
               : "memory");
  return v;
}

// ------------------------------------------------------------ bulk copy --

// Global -> shared bulk copy through the TMA engine; completion is signalled
// as transaction bytes on `bar`.  16-byte aligned addresses, size % 16 == 0.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// Shared (this CTA) -> shared (CTA of the cluster) bulk copy; completion is
// signalled as transaction bytes on the destination CTA's mbarrier.
__device__ __forceinline__ void bulk_s2cluster(uint32_t dst_cluster, uint32_t src_cta, uint32_t bytes,
                                               uint32_t bar_cluster) {
  asm volatile(
      "cp.async.bulk.shared::cluster.shared::cta.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          dst_cluster),
      "r"(src_cta), "r"(bytes), "r"(bar_cluster)
      : "memory");
}
__device__ __forceinline__ void bulk_commit_group() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// wait until every committed bulk copy of this thread has read its source
__device__ __forceinline__ void bulk_wait_read_all() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ------------------------------------------------------------ tcgen05 ----

__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
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
// arrive on `bar` once all previously issued tcgen05 ops of this thread finish
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}

// Shared-memory matrix descriptor (sm_100 format): start address, leading and
// stride byte offsets (16-byte units), descriptor version 1 (bits 46-47) and
// the swizzle mode in bits 61-63 (0 none, 2 = 128-byte, 4 = 64-byte).
enum : uint64_t { kSwNone = 0, kSw128 = 2, kSw64 = 4 };
__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo, uint64_t swz) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (swz << 61);
}

// Instruction descriptor of kind::mxf4nvf4 (block-scaled E2M1 x E2M1 with
// E4M3 scales, FP32 accumulate): A/B format E2M1 (1) in bits 7-9 / 10-12,
// K-major A and B, N >> 3 in bits 17-22, M >> 4 in bits 24-28, sparse flag
// in bit 2.
__host__ __device__ constexpr uint32_t idesc_nvf4(int M, int N, bool sparse) {
  return (sparse ? (1u << 2) : 0u) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) |
         ((uint32_t)(M >> 4) << 24);
}

// Instruction descriptor of kind::mxf4 (E2M1 x E2M1 with E8M0 scales, one
// per 32 stored elements -- 64 logical K in the sparse form -- FP32
// accumulate): the fields of idesc_nvf4 plus the scale format (bit 23 = E8M0)
// and the scale-factor IDs, A in bits 29-30 and B in bits 4-5: the byte of
// the 32-bit TMEM scale column where this MMA's two scales per row start.
__host__ __device__ constexpr uint32_t idesc_mxf4(int M, int N, bool sparse, uint32_t a_id, uint32_t b_id) {
  return (sparse ? (1u << 2) : 0u) | (b_id << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) |
         (1u << 23) | ((uint32_t)(M >> 4) << 24) | (a_id << 29);
}

// smem (described by desc) -> TMEM: 128 lanes x 16 bytes
__device__ __forceinline__ void tc_cp_128x128b(uint32_t taddr, uint64_t desc) {
  asm volatile("tcgen05.cp.cta_group::1.128x128b [%0], %1;" ::"r"(taddr), "l"(desc) : "memory");
}
// smem -> TMEM: 32 lanes x 16 bytes, replicated into all four lane quarters
__device__ __forceinline__ void tc_cp_32x128b_x4(uint32_t taddr, uint64_t desc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(desc) : "memory");
}

// D(tmem) (+)= A(smem) x B(smem) with per-16 E4M3 block scales from TMEM
__device__ __forceinline__ void mma_nvf4(uint32_t d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         uint32_t sfa, uint32_t sfb, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
      : "memory");
}
// Sparse variant: A is the 2:1 compressed operand, metadata in TMEM at `e`.
__device__ __forceinline__ void mma_sp_nvf4(uint32_t d, uint64_t adesc, uint64_t bdesc, uint32_t e,
                                            uint32_t idesc, uint32_t sfa, uint32_t sfb,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %5, 0;\n\t"
      "tcgen05.mma.sp.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, [%3], %4, [%6], [%7], "
      "p;\n\t}" ::"r"(d),
      "l"(adesc), "l"(bdesc), "r"(e), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
      : "memory");
}

// MXFP4 forms: per-32 (sparse: per-64 logical) E8M0 scales from TMEM; the
// scale addresses carry the scale-factor ID in bits 30-31 as well
__device__ __forceinline__ void mma_mxf4(uint32_t d, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t sfa,
                                         uint32_t sfb, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf4.block_scale.block32 [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
      : "memory");
}
__device__ __forceinline__ void mma_sp_mxf4(uint32_t d, uint64_t adesc, uint64_t bdesc, uint32_t e, uint32_t idesc,
                                            uint32_t sfa, uint32_t sfb, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %5, 0;\n\t"
      "tcgen05.mma.sp.cta_group::1.kind::mxf4.block_scale.block32 [%0], %1, %2, [%3], %4, [%6], [%7], "
      "p;\n\t}" ::"r"(d),
      "l"(adesc), "l"(bdesc), "r"(e), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
      : "memory");
}

// ---------------------------------------------- tcgen05, CTA pairs ----
// The cta_group::2 forms: two CTAs of a cluster (ranks 2i, 2i+1) act as one
// MMA unit.  One thread of the even CTA issues the MMAs and copies for both;
// each CTA keeps its own rows of A, its half of B's rows and its own rows of
// the accumulator, at the same shared-memory and TMEM addresses in both.  A
// kernel uses one cta_group throughout.

// collective over the pair: the same warp of both CTAs allocates the same
// columns in both TMEMs, each writing the address to its own shared memory
__device__ __forceinline__ void tmem_alloc_pair(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
// arrive on `bar` of this CTA once the pair ops this thread issued finish
__device__ __forceinline__ void tc_commit_pair(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}
// ... on the barrier at the same offset in every CTA of cta_mask
__device__ __forceinline__ void tc_commit_pair_mc(uint64_t* bar, uint16_t cta_mask) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::
                   "r"(smem_u32(bar)),
               "h"(cta_mask)
               : "memory");
}
// each CTA's shared memory (same offset) -> its own TMEM, as the 1-CTA forms
__device__ __forceinline__ void tc_cp_pair_128x128b(uint32_t taddr, uint64_t desc) {
  asm volatile("tcgen05.cp.cta_group::2.128x128b [%0], %1;" ::"r"(taddr), "l"(desc) : "memory");
}
__device__ __forceinline__ void tc_cp_pair_32x128b_x4(uint32_t taddr, uint64_t desc) {
  asm volatile("tcgen05.cp.cta_group::2.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(desc) : "memory");
}
// D (M = 256 over the pair) (+)= A x B, per-16 E4M3 block scales from TMEM
__device__ __forceinline__ void mma_pair_nvf4(uint32_t d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                              uint32_t sfa, uint32_t sfb, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
      : "memory");
}
__device__ __forceinline__ void mma_pair_sp_nvf4(uint32_t d, uint64_t adesc, uint64_t bdesc, uint32_t e,
                                                 uint32_t idesc, uint32_t sfa, uint32_t sfb, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %5, 0;\n\t"
      "tcgen05.mma.sp.cta_group::2.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, [%3], %4, [%6], [%7], "
      "p;\n\t}" ::"r"(d),
      "l"(adesc), "l"(bdesc), "r"(e), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
      : "memory");
}

// TMEM -> registers: this thread's lane, 32 consecutive 32-bit columns
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
__device__ __forceinline__ void tmem_ld_wait() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

}  // namespace sharq
