// gemm.cu - sharq_linear / sharq_linear_grouped: the dual-path FP4 GEMM.
//
// xllm-io review of SharQ, section 3.4:
//   Y = GEMM_sp(Q_sp(X_sp), Q_w,sp(W)) + GEMM_dn(Q_dn(R), Q_w,dn(W))
// and section 3.5 ("residual accumulation: the dense branch accumulates
// directly into the sparse branch's output, no second full branch is
// materialised"; "shared FP4 weight payload ... path-specific scale views").
//
// B200 design (one CTA per 128 x BN output tile, warp-specialised):
//   warp 0      producer: per 256-K stage, bulk copies (TMA engine) of the
//               pre-tiled operands -- backbone codes, metadata, residual
//               codes, their scales, the weight codes and both weight scale
//               views -- into a STAGES-deep shared-memory ring, completion
//               tracked by mbarrier transaction bytes.
//   warp 1      TMEM allocation; one elected thread issues, per stage,
//               2 sparse block-scaled FP4 MMAs (tcgen05.mma.sp
//               kind::mxf4nvf4, K=128 logical each, one scale per 32 logical
//               K) and 4 dense ones (kind::mxf4nvf4 block16, K=64 each), all
//               into ONE fp32 TMEM accumulator and all reading the SAME
//               weight tile in shared memory; tcgen05.commit releases the
//               stage.
//   warps 2-5   epilogue: tcgen05.ld of the accumulator (one row per thread),
//               y = f32(acc * f32(s_g * s_w)), bf16 or fp32 stores.
//   warps 6-    copy warps: tcgen05.cp of the stage's metadata and scale
//               factors into TMEM, spread over 2-4 warps.  A tcgen05.cp costs
//               about as long as an MMA to issue from one thread, whatever
//               its size, and copies from different warps proceed side by
//               side, so the copies of later stages run while the MMAs of
//               stage i do.  Each ring slot has its own TMEM scale region, so
//               a stage's copies start as soon as its data has landed (a
//               copy's completion takes a good fraction of a microsecond);
//               each copy warp commits to the slot's mbarrier, which the MMA
//               thread waits on.
// Prefill shapes with at least two 128-row tiles run on CTA pairs instead
// (tcgen05 cta_group::2, 256 x 256 tiles; roles at sharq_gemm_pair_kernel).
// Split-K (decode shapes, where output tiles alone cannot fill 148 SMs):
// the S CTAs that share an output tile form one thread-block cluster
// (1 x 1 x S); each takes a contiguous range of K stages.  CTA r of the
// cluster owns 1/S of the tile's valid rows: every CTA pushes that slice of
// its fp32 partial, row by row from registers, into a receive buffer in the
// owner's shared memory over distributed shared memory (st.async stores that
// complete the owner's barrier by transaction bytes), and the owner sums the
// S slices in rank order -- deterministic, no global scratch, no atomics,
// one bounded wait.
// Rows beyond the activation's valid rows are not copied into shared memory
// (decode: T = 1 moves 1 row of codes, not 128) -- sharq_prep does not even
// write them; their accumulator rows hold garbage that is never stored (MMA
// rows are independent), and their metadata is set to a valid pattern in
// shared memory once at start-up.
// Every wait is bounded by the global timer; on timeout the CTA records
// SHARQ_ERR_TIMEOUT in the workspace error word and leaves.
#include <stdlib.h>

#include "quant.cuh"

namespace sharq {

namespace {

// 6 warps (producer, MMA, 4 epilogue) + the copy warps
constexpr int kBaseThreads = 192;
__host__ __device__ constexpr int gemm_threads(int copy_warps) { return kBaseThreads + 32 * copy_warps; }

// Optional phase timeline (compile with -DSHARQ_TRACE): 16 global-timer
// stamps per CTA -- entry, set-up done, first stage issued, first stage
// consumed, last MMA committed, accumulator ready, epilogue done, exit; in the
// fused form also: dependency resolved, 1/rms known, s_g known, first and
// last activation stage written.
#ifdef SHARQ_TRACE
__device__ unsigned long long* g_trace = nullptr;
#define TRACE_POINT(k)                                                                                   \
  do {                                                                                                   \
    if (g_trace)                                                                                         \
      g_trace[(((size_t)blockIdx.z * gridDim.y + blockIdx.y) * gridDim.x + blockIdx.x) * 16 + (k)] =     \
          globaltimer_ns();                                                                              \
  } while (0)
#else
#define TRACE_POINT(k) \
  do {                 \
  } while (0)
#endif
constexpr uint64_t kWaitLimitNs = 4000000000ull;  // 4 s: far beyond any tile's work
constexpr int kErrTimeout = -5;
constexpr int kErrInvalid = -1;

struct GemmArgs {
  const uint8_t* a_sp;
  const uint8_t* a_meta;
  const uint8_t* a_spsf;
  const uint8_t* a_r;
  const uint8_t* a_rsf;
  const uint8_t* a_rmeta;  // Sparse+Sparse: the residual's metadata
  const float* s_g;
  const uint8_t* w_codes;
  const uint8_t* w_sf32;
  const uint8_t* w_sf16;
  const float* s_w;
  void* Y;
  const int* group_offsets;  // device [E+1] or nullptr
  int* err;                  // workspace error word or nullptr
  const int* act_err;        // error word left by sharq_prep (propagated)
  int T, K, D, E;
  int out_f32;
  int sharq_mode;
  int splits;
  int per_token;  // s_g holds one scale per activation row
  // persistent / pair tile order: 0 = row-tile major (consecutive tiles share
  // activation rows), 1 = column-tile major (consecutive tiles share weight
  // columns); the launcher picks the order that keeps the smaller operand in L2
  int n_major;
  // fused decode form: raw activations are prepared inside the GEMM
  const __nv_bfloat16* X;      // [T][K] bf16
  const __nv_bfloat16* gamma;  // [K] bf16 or nullptr
  float eps;
};

template <int BN, bool kSplit, bool kFused = false>
struct Cfg {
  static constexpr int kHalves = BN / 128;
  // copy warps: 4 where registers allow (65536 / threads per thread), 2 for
  // the register-heavy fused form
  static constexpr int kCW = kFused ? 2 : 4;
  static constexpr int kThreadsT = gemm_threads(kCW);
  // split-K CTAs do few stages and need room for the received partial rows
  static constexpr int kStages = (kSplit || BN == 256) ? 3 : 4;
  // shared-memory stage layout (bytes); 1024-aligned where a swizzle needs it
  static constexpr int kOffB = 0;
  static constexpr int kOffAR = kOffB + BN * 128;
  static constexpr int kOffASP = kOffAR + kCodesTile;
  static constexpr int kOffE = kOffASP + kSpTile;
  static constexpr int kOffSFASP = kOffE + kMetaTile;
  static constexpr int kOffSFAR = kOffSFASP + kSf32Tile;
  static constexpr int kOffSFB32 = kOffSFAR + kSf16Tile;
  static constexpr int kOffSFB16 = kOffSFB32 + kHalves * kSf32Tile;
  static constexpr int kStageBytes = kOffSFB16 + kHalves * kSf16Tile;
  static constexpr int kRingBytes = kStages * kStageBytes;
  // split-K receive buffer (outside the ring, so peers may write into it
  // while this CTA's own mainloop still runs): S slices of ceil(rows/S) rows
  static constexpr int kRowFloats = BN + 4;  // padded: conflict-free float4 access
  // receive buffer: S slices of ceil(rows / S) + 1 rows x BN floats, at most
  // (128 + 2 S - 1) x 512 bytes for S <= 4
  static constexpr int kRecvRows = 136;
  static constexpr int kRecvBytes = kSplit ? kRecvRows * kRowFloats * 4 : 0;
  static constexpr int kSmemBytes = kRingBytes + kRecvBytes + 1024;
  // TMEM columns: the accumulator, then one region of metadata + scale
  // factors per ring slot (a slot is refilled only after the MMAs that read
  // its region have completed).
  static constexpr uint32_t kColAcc = 0;
  static constexpr uint32_t kSfbCols = BN / 32;  // per MMA: one column per 32 rows of B
  static constexpr uint32_t kSfE = 0, kSfASP = 8, kSfAR = 16, kSfB32 = 32, kSfB16 = 32 + 2 * kSfbCols;
  static constexpr uint32_t kSfRegion = 32 + 6 * kSfbCols;
  static constexpr uint32_t kColSf0 = BN;
  static constexpr uint32_t kColsUsed = BN + kStages * kSfRegion;
  static constexpr uint32_t kTmemCols = kColsUsed <= 256 ? 256 : 512;
  // transaction bytes per stage (activation code copies trimmed to valid rows)
  static constexpr uint32_t kTxSharq = BN * 128 + kHalves * (kSf32Tile + kSf16Tile) + kCodesTile + kSpTile +
                                       kMetaTile + kSf32Tile + kSf16Tile;
  static constexpr uint32_t kTxNvfp4 = BN * 128 + kHalves * kSf16Tile + kCodesTile + kSf16Tile;
  static constexpr uint32_t kTxB = BN * 128 + kHalves * (kSf32Tile + kSf16Tile);  // weight side only
  static_assert(kStageBytes % 1024 == 0, "stage must keep 1024-byte alignment");
  static_assert(kColsUsed <= 512, "TMEM overflow");
  static_assert(kSmemBytes <= 232448, "shared memory overflow");
  static_assert(!kSplit || BN == 128, "split-K uses 128-wide tiles");
  static_assert(!kSplit || kRecvBytes >= (128 + 2 * 4 - 1) * (BN / 4) * 16, "split-K receive buffer");
};

__device__ __forceinline__ void record_error(int* err, int code) {
  if (err) atomicCAS(err, 0, code);
}

// y = f32(acc * scale), 32 consecutive columns of one row, bf16 or fp32
__device__ __forceinline__ void store_row32(void* Y, int out_f32, size_t off, const uint32_t (&v)[32], float scale) {
  if (out_f32) {
    float* y = static_cast<float*>(Y) + off;
#pragma unroll
    for (int i = 0; i < 32; i += 4)
      *reinterpret_cast<float4*>(y + i) =
          make_float4(__fmul_rn(__uint_as_float(v[i]), scale), __fmul_rn(__uint_as_float(v[i + 1]), scale),
                      __fmul_rn(__uint_as_float(v[i + 2]), scale), __fmul_rn(__uint_as_float(v[i + 3]), scale));
  } else {
    __nv_bfloat16* y = static_cast<__nv_bfloat16*>(Y) + off;
#pragma unroll
    for (int i = 0; i < 32; i += 8) {
      uint4 pk;
      uint32_t* w = reinterpret_cast<uint32_t*>(&pk);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        __nv_bfloat162 b2 = __floats2bfloat162_rn(__fmul_rn(__uint_as_float(v[i + 2 * k]), scale),
                                                  __fmul_rn(__uint_as_float(v[i + 2 * k + 1]), scale));
        w[k] = *reinterpret_cast<uint32_t*>(&b2);
      }
      *reinterpret_cast<uint4*>(y + i) = pk;
    }
  }
}

__device__ __forceinline__ void store4(void* Y, int out_f32, size_t off, float4 a, float scale) {
  const float x = __fmul_rn(a.x, scale), y = __fmul_rn(a.y, scale), z = __fmul_rn(a.z, scale),
              w = __fmul_rn(a.w, scale);
  if (out_f32) {
    *reinterpret_cast<float4*>(static_cast<float*>(Y) + off) = make_float4(x, y, z, w);
  } else {
    __nv_bfloat162 lo = __floats2bfloat162_rn(x, y), hi = __floats2bfloat162_rn(z, w);
    uint2 pk;
    pk.x = *reinterpret_cast<uint32_t*>(&lo);
    pk.y = *reinterpret_cast<uint32_t*>(&hi);
    *reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(Y) + off) = pk;
  }
}

// Global stores of a warp's 32 output rows (row = lane, kCols bf16 columns
// held as packed pairs pk) through the warp's 4 KB of shared memory, 64
// columns (128 bytes of each row) at a time: stored straight from registers a
// warp instruction would touch 32 rows' lines, here it writes 4 whole 128-byte
// lines.  Chunk q of row r sits at q ^ (r % 8) so both the writes and the
// reads spread over all banks.  y0: row 0 of the warp, first column; ld: the
// row stride (elements); rows: the warp's valid rows (the others are not
// stored).
template <int kCols>
__device__ __forceinline__ void store_rows_bf16_staged(const uint32_t (&pk)[kCols / 2], uint8_t* wst,
                                                       __nv_bfloat16* y0, size_t ld, int rows, int lane) {
  const int rsub = lane >> 3, q = lane & 7;  // store phase: row within a group of 4, 16-byte chunk
#pragma unroll
  for (int c = 0; c < kCols / 64; ++c) {
#pragma unroll
    for (int j = 0; j < 8; ++j)
      *reinterpret_cast<uint4*>(wst + lane * 128 + ((j ^ (lane & 7)) << 4)) =
          make_uint4(pk[32 * c + 4 * j], pk[32 * c + 4 * j + 1], pk[32 * c + 4 * j + 2], pk[32 * c + 4 * j + 3]);
    __syncwarp();
#pragma unroll
    for (int it = 0; it < 8; ++it) {
      const int r = 4 * it + rsub;
      if (r < rows)
        *reinterpret_cast<uint4*>(y0 + (size_t)r * ld + 64 * c + 8 * q) =
            *reinterpret_cast<const uint4*>(wst + r * 128 + ((q ^ (r & 7)) << 4));
    }
    __syncwarp();
  }
}

// Expert that owns m-tile mt in the grouped form (offsets are 128-row
// aligned), 0 without groups, -1 if the offsets do not cover the tile.
__device__ __forceinline__ int tile_expert(const GemmArgs& args, int mt) {
  if (!args.group_offsets) return 0;
  const int row0 = mt * 128;
  int e = -1;
  int lo = 0, hi = args.E - 1;
  while (lo <= hi) {
    const int mid = (lo + hi) >> 1;
    if (args.group_offsets[mid] <= row0) {
      e = mid;
      lo = mid + 1;
    } else {
      hi = mid - 1;
    }
  }
  while (e >= 0 && e < args.E && args.group_offsets[e + 1] <= row0) ++e;
  if (e < 0 || e >= args.E || args.group_offsets[e] > row0 || args.group_offsets[e + 1] <= row0) e = -1;
  return e;
}

// (row tile, column tile) of persistent tile index `tile` over m_tiles x
// n_tiles tiles.  Row-major order suits operands whose activation side is the
// larger (each weight column tile is revisited while the whole weight stays in
// L2); column-major order suits a weight larger than the activation, e.g. a
// wide gate+up projection whose 80 MB weight would otherwise be evicted by the
// output stream before the next row tile comes back to it.
__device__ __forceinline__ void tile_coords(int tile, int m_tiles, int n_tiles, int n_major, int& mt, int& nt) {
  if (n_major) {
    nt = tile / m_tiles;
    mt = tile - nt * m_tiles;
  } else {
    mt = tile / n_tiles;
    nt = tile - mt * n_tiles;
  }
}

// Programmatic dependent launch: wait until the preceding grid in the stream
// has completed and its memory is visible (returns at once if there is none).
__device__ __forceinline__ void grid_dependency_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// 16-byte store into a peer CTA's shared memory that counts its bytes on the
// peer's mbarrier (transaction bytes) when it lands: no release fence and no
// separate arrival are needed for the peer to see it.
__device__ __forceinline__ void st_async_f4(uint32_t addr, float a, float b, float c, float d, uint32_t remote_bar) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.f32 [%0], {%1, %2, %3, %4}, [%5];" ::"r"(addr),
               "f"(a), "f"(b), "f"(c), "f"(d), "r"(remote_bar)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive_local(uint64_t* bar) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void epi_barrier() {  // the 128 epilogue threads
  asm volatile("bar.sync 1, 128;" ::: "memory");
}

__device__ __forceinline__ void st_cluster_f64(uint32_t addr, double v) {
  asm volatile("st.shared::cluster.f64 [%0], %1;" ::"r"(addr), "d"(v) : "memory");
}
__device__ __forceinline__ void st_cluster_f32(uint32_t addr, float v) {
  asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(addr), "f"(v) : "memory");
}

// Sum, across the 32 lanes, eight per-lane values at once (a transposing
// butterfly: 9 double shuffles instead of 40).  Lane l returns the total of
// value (l >> 2) & 7.
__device__ __forceinline__ double warp_sum8(double (&v)[8], int lane) {
  const bool b4 = lane & 16, b3 = lane & 8, b2 = lane & 4;
  double w4[4], w2[2];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const double send = b4 ? v[j] : v[j + 4];
    const double keep = b4 ? v[j + 4] : v[j];
    w4[j] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
  }
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    const double send = b3 ? w4[j] : w4[j + 2];
    const double keep = b3 ? w4[j + 2] : w4[j];
    w2[j] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
  }
  double w = (b2 ? w2[1] : w2[0]) + __shfl_xor_sync(0xffffffffu, b2 ? w2[0] : w2[1], 4);
  w += __shfl_xor_sync(0xffffffffu, w, 2);
  w += __shfl_xor_sync(0xffffffffu, w, 1);
  return w;
}

// Shared state of the fused decode form's statistics exchange.
template <bool kSplit>
struct FusedStats {
  double part[4][32];                // per epilogue warp, per row: sum of squares over this CTA's K-slice
  double ss[kSplit ? 8 : 1][32];     // per cluster rank, per row (written by the peers)
  float mx[kSplit ? 8 : 1];          // per cluster rank: max |Xn| over its K-slice
  float inv[32];                     // 1/rms per row
  float wmax[4];
  float s;                           // the per-tensor scale s_g
};

// bounded wait on a barrier that peers of the cluster arrive on
__device__ __forceinline__ bool cluster_bar_wait(uint64_t* bar, uint64_t deadline, volatile int* abort) {
  while (!mbar_try_wait_cluster(bar, 0)) {
    if (*abort || globaltimer_ns() > deadline) return false;
  }
  return true;
}

// The epilogue warps' prep phase of the fused decode form (128 threads,
// T <= 32 rows, this CTA's K-slice of ks tiles [ks0, ks0 + nks)).
//  1. sum of squares of every row over the K-slice (fp64), exchanged with the
//     S - 1 other CTAs of the cluster, which hold the rest of K; every CTA
//     adds the S partials in rank order -> identical 1/rms everywhere;
//  2. max |Xn| over the K-slice, exchanged the same way -> s_g;
//  3. the A half of every stage of the K-slice, in the MMA layout.
// Loads are issued eight rows at a time, so each warp keeps eight 16-byte
// loads in flight instead of walking whole rows one load after another.
template <class C, bool kSplit>
__device__ __forceinline__ bool fused_prep(const GemmArgs& args, uint8_t* smem, int ks0, int nks, int T, int S,
                                           uint64_t deadline, volatile int* abort, uint64_t* empty_bar,
                                           uint64_t* afull_bar, uint64_t* stat_bar, FusedStats<kSplit>& fs) {
  const int ew = (threadIdx.x >> 5) - 2, lane = threadIdx.x & 31;
  const int K = args.K;
  const uint32_t rank = kSplit ? cluster_ctarank() : 0u;
  const __nv_bfloat16* Xs = args.X + (size_t)ks0 * 256 + lane * 8;  // this lane's column in tile 0 of the slice
  grid_dependency_wait();  // X comes from the preceding kernel
  if (threadIdx.x == 64) TRACE_POINT(8);
  // ---- 1. sums of squares -> 1/rms
  if (args.gamma) {
    for (int r0 = 0; r0 < T; r0 += 8) {
      double acc[8];
#pragma unroll
      for (int g = 0; g < 8; ++g) acc[g] = 0.0;
#pragma unroll 2
      for (int i = ew; i < nks; i += 4) {
        uint4 raw[8];
#pragma unroll
        for (int g = 0; g < 8; ++g)
          raw[g] = r0 + g < T ? *reinterpret_cast<const uint4*>(Xs + (size_t)(r0 + g) * K + i * 256)
                              : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
        for (int g = 0; g < 8; ++g) {
          float f[8];
          bf16x8_to_float(raw[g], f);
#pragma unroll
          for (int e = 0; e < 8; ++e) acc[g] += (double)f[e] * (double)f[e];
        }
      }
      const double tot = warp_sum8(acc, lane);
      const int r = r0 + ((lane >> 2) & 7);
      if ((lane & 3) == 0 && r < T) fs.part[ew][r] = tot;
    }
    epi_barrier();
    if (ew == 0 && lane < T) {
      const double ps = ((fs.part[0][lane] + fs.part[1][lane]) + fs.part[2][lane]) + fs.part[3][lane];
      if (kSplit) {
        const uint32_t dst = smem_u32(&fs.ss[rank][lane]);
        for (int p = 0; p < S; ++p) st_cluster_f64(mapa_shared(dst, (uint32_t)p), ps);
        // each row's sender releases its own stores: S x T arrivals per CTA
        for (int p = 0; p < S; ++p) mbar_arrive_remote(mapa_shared(smem_u32(&stat_bar[0]), (uint32_t)p));
      } else {
        fs.ss[0][lane] = ps;
      }
    }
    if (kSplit) {
      if (!cluster_bar_wait(&stat_bar[0], deadline, abort)) return false;
    } else {
      epi_barrier();
    }
    if (ew == 0 && lane < T) {
      double tot = fs.ss[0][lane];
      for (int p = 1; p < (kSplit ? S : 1); ++p) tot += fs.ss[p][lane];
      fs.inv[lane] = (float)(1.0 / sqrt(tot / (double)K + (double)args.eps));
    }
  } else if (ew == 0 && lane < T) {
    fs.inv[lane] = 1.0f;
  }
  epi_barrier();
  if (threadIdx.x == 64) TRACE_POINT(9);
  // ---- 2. max |Xn| over the slice -> s_g
  float m = 0.0f;
  const __nv_bfloat16* Gs = args.gamma ? args.gamma + (size_t)ks0 * 256 + lane * 8 : nullptr;
  for (int r0 = 0; r0 < T; r0 += 8) {
#pragma unroll 2
    for (int i = ew; i < nks; i += 4) {
      uint4 raw[8];
#pragma unroll
      for (int g = 0; g < 8; ++g)
        raw[g] = r0 + g < T ? *reinterpret_cast<const uint4*>(Xs + (size_t)(r0 + g) * K + i * 256)
                            : make_uint4(0u, 0u, 0u, 0u);
      float gm[8];
      if (Gs) bf16x8_to_float(*reinterpret_cast<const uint4*>(Gs + i * 256), gm);
#pragma unroll
      for (int g = 0; g < 8; ++g) {
        float f[8];
        bf16x8_to_float(raw[g], f);
        const float inv = fs.inv[min(r0 + g, T - 1)];
#pragma unroll
        for (int e = 0; e < 8; ++e) m = fmaxf(m, fabsf(Gs ? norm_one(f[e], inv, gm[e]) : f[e]));
      }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if (lane == 0) fs.wmax[ew] = m;
  epi_barrier();
  if (threadIdx.x == 64) {
    const float cm = fmaxf(fmaxf(fs.wmax[0], fs.wmax[1]), fmaxf(fs.wmax[2], fs.wmax[3]));
    if (kSplit) {
      const uint32_t dst = smem_u32(&fs.mx[rank]);
      for (int p = 0; p < S; ++p) st_cluster_f32(mapa_shared(dst, (uint32_t)p), cm);
      for (int p = 0; p < S; ++p) mbar_arrive_remote(mapa_shared(smem_u32(&stat_bar[1]), (uint32_t)p));
    } else {
      fs.mx[0] = cm;
    }
  }
  if (kSplit) {
    if (!cluster_bar_wait(&stat_bar[1], deadline, abort)) return false;
  } else {
    epi_barrier();
  }
  float gmax = fs.mx[0];
  for (int p = 1; p < (kSplit ? S : 1); ++p) gmax = fmaxf(gmax, fs.mx[p]);
  const float s = gmax > 0.0f ? __fdiv_rn(gmax, kGlobalDiv) : 1.0f;
  const float six_s = __fmul_rn(6.0f, s);
  if (threadIdx.x == 64) {
    fs.s = s;
    TRACE_POINT(10);
  }
  // ---- 3. the A half of every stage of this CTA's K-slice (rows ew, ew+4, ...)
  for (int i = 0; i < nks; ++i) {
    const int st = i % C::kStages;
    uint4 raw[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int r = ew + 4 * j;
      raw[j] = r < T ? *reinterpret_cast<const uint4*>(Xs + (size_t)r * K + i * 256) : make_uint4(0u, 0u, 0u, 0u);
    }
    float gm[8];
    if (Gs) bf16x8_to_float(*reinterpret_cast<const uint4*>(Gs + i * 256), gm);
    if (i >= C::kStages && !mbar_wait(&empty_bar[st], ((i / C::kStages) & 1) ^ 1, deadline, abort)) return false;
    uint8_t* base = smem + st * C::kStageBytes;
    const QuantPtrs q{base + C::kOffASP, base + C::kOffE, base + C::kOffSFASP, base + C::kOffAR, base + C::kOffSFAR};
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int r = ew + 4 * j;
      if (r < T) {
        float x[8];
        bf16x8_to_float(raw[j], x);
        if (Gs) {
          const float inv = fs.inv[r];
#pragma unroll
          for (int e = 0; e < 8; ++e) x[e] = norm_one(x[e], inv, gm[e]);
        }
        quant_runs<1, kKindSharq>(x, r, lane, 256, s, six_s, q);  // one 256-K tile: tile index 0
      }
    }
    fence_proxy_async_smem();   // generic writes -> visible to tcgen05.cp / MMA
    mbar_arrive_local(&afull_bar[st]);
    if (threadIdx.x == 64 && (i == 0 || i == nks - 1)) TRACE_POINT(i == 0 ? 11 : 12);
  }
  return true;
}

// The stage's copies into the TMEM scale region sf, weight side then
// activation side (copy number n is issued by copy warp n % kCW; the
// counter n runs on across both calls).
template <class C>
__device__ __forceinline__ void copies_weight(uint32_t st, uint32_t sf, bool sharq, int cw, int& n) {
#pragma unroll
  for (int j = 0; j < 4; ++j)
#pragma unroll
    for (int h = 0; h < C::kHalves; ++h)
      if (n++ % C::kCW == cw)
        tc_cp_32x128b_x4(sf + C::kSfB16 + j * C::kSfbCols + 4 * h,
                         smem_desc(st + C::kOffSFB16 + h * kSf16Tile + 512 * j, 0, 128, kSwNone));
  if (sharq) {
#pragma unroll
    for (int j = 0; j < 2; ++j)
#pragma unroll
      for (int h = 0; h < C::kHalves; ++h)
        if (n++ % C::kCW == cw)
          tc_cp_32x128b_x4(sf + C::kSfB32 + j * C::kSfbCols + 4 * h,
                           smem_desc(st + C::kOffSFB32 + h * kSf32Tile + 512 * j, 0, 128, kSwNone));
  }
}
template <class C>
__device__ __forceinline__ void copies_act(uint32_t st, uint32_t sf, bool sharq, int cw, int& n) {
#pragma unroll
  for (int j = 0; j < 4; ++j)
    if (n++ % C::kCW == cw)
      tc_cp_32x128b_x4(sf + C::kSfAR + 4 * j, smem_desc(st + C::kOffSFAR + 512 * j, 0, 128, kSwNone));
  if (sharq) {
    if (n++ % C::kCW == cw) tc_cp_128x128b(sf + C::kSfE, smem_desc(st + C::kOffE, 0, 128, kSwNone));
#pragma unroll
    for (int j = 0; j < 2; ++j)
      if (n++ % C::kCW == cw)
        tc_cp_32x128b_x4(sf + C::kSfASP + 4 * j, smem_desc(st + C::kOffSFASP + 512 * j, 0, 128, kSwNone));
  }
}

// kFused: the decode form that prepares the activation itself.  The S CTAs
// of a cluster split K between them: each reduces the row sums of squares and
// the |Xn| max over its own K-slice and the partials are exchanged over
// distributed shared memory (combined in rank order, so every CTA of every
// cluster derives the same 1/rms and s_g); each CTA then quantizes its own
// K-slice straight into the A half of each shared-memory stage, in the MMA
// layout, while the producer streams the weight half.  No prepared activation
// goes through HBM and no separate prep kernel runs.
template <int BN, bool kSplit, bool kFused>
__global__ void __launch_bounds__(Cfg<BN, kSplit, kFused>::kThreadsT, 1) sharq_gemm_kernel(const GemmArgs args) {
  using C = Cfg<BN, kSplit, kFused>;
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full_bar[C::kStages];
  __shared__ __align__(8) uint64_t empty_bar[C::kStages];
  __shared__ __align__(8) uint64_t acc_bar;
  __shared__ __align__(8) uint64_t recv_bar;
  __shared__ __align__(8) uint64_t afull_bar[kFused ? C::kStages : 1];
  __shared__ __align__(8) uint64_t sf_full[C::kStages];  // ring slot s: its stage's copies have landed
  __shared__ __align__(8) uint64_t cp_fin[C::kCW];   // each copy warp's last copies
  __shared__ uint32_t tmem_base_sh;
  __shared__ volatile int abort_sh;
  __shared__ int expert_sh;
  __shared__ __align__(8) uint64_t stat_bar[2];
  __shared__ __align__(8) FusedStats<kSplit> fstats;

  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nt = blockIdx.x, mt = blockIdx.y, split = blockIdx.z;
  const int KS = args.K >> 8;
  const int S = kSplit ? args.splits : 1;
  const int ks0 = (int)(((long long)split * KS) / S);
  const int ks1 = (int)(((long long)(split + 1) * KS) / S);
  const int nks = ks1 - ks0;
  const int NB = args.D >> 7;
  const int valid = min(128, args.T - mt * 128);  // rows of this m-tile that exist
  // split-K: CTA r of the cluster owns rows [r*rows_per, r*rows_per + my_n)
  const int rows_per = (valid + S - 1) / S;
  const int my0 = split * rows_per;
  const int my_n = max(0, min(valid, my0 + rows_per) - my0);
  const uint64_t deadline = globaltimer_ns() + kWaitLimitNs;
  if (threadIdx.x == 0) TRACE_POINT(0);

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    mbar_init(&acc_bar, 1);
    for (int st = 0; st < C::kStages; ++st) mbar_init(&sf_full[st], C::kCW);
    for (int c = 0; c < C::kCW; ++c) mbar_init(&cp_fin[c], 1);
    if (kFused) {
      for (int st = 0; st < C::kStages; ++st) mbar_init(&afull_bar[st], 128);  // the epilogue threads
      // statistics exchange: every CTA of the cluster arrives once per row,
      // then once for the max
      mbar_init(&stat_bar[0], (uint32_t)(S * max(valid, 1)));
      mbar_init(&stat_bar[1], (uint32_t)S);
    }
    mbar_init(&recv_bar, 1u);
    fence_mbar_init();
    // the receive barrier completes when all S senders' rows have landed
    // (transaction bytes of their st.async stores); set before the cluster
    // sync below, so before any peer can store
    if (kSplit && my_n > 0) mbar_arrive_expect_tx(&recv_bar, (uint32_t)(S * my_n * BN * 4));
    abort_sh = 0;
    expert_sh = tile_expert(args, mt);
  }
  if (warp == 1) {
    tmem_alloc(&tmem_base_sh, C::kTmemCols);
    tmem_relinquish();
  }
  if (args.sharq_mode && valid < 128) {
    // Rows past the activation's end are never copied in; give their
    // metadata a valid pattern (pairs 0 and 1) once, in every stage.
    for (int idx = threadIdx.x; idx < C::kStages * (128 - valid); idx += C::kThreadsT) {
      const int st = idx / (128 - valid), row = valid + idx % (128 - valid);
      *reinterpret_cast<uint4*>(smem + st * C::kStageBytes + C::kOffE + row * 16) =
          make_uint4(0x44444444u, 0x44444444u, 0x44444444u, 0x44444444u);
    }
    fence_proxy_async_smem();  // visible to tcgen05.cp (async proxy)
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (kSplit) cluster_sync_all();  // peers' barriers initialised before any remote traffic
  if (threadIdx.x == 0) TRACE_POINT(1);
  const uint32_t tmem = tmem_base_sh;
  const int expert = expert_sh;
  if (expert < 0) {  // (never in split mode: no groups there)
    if (threadIdx.x == 0) record_error(args.err, kErrInvalid);
    __syncthreads();
    if (warp == 1) tmem_dealloc(tmem, C::kTmemCols);
    return;
  }
  const bool sharq = args.sharq_mode != 0;

  if (warp == 0) {
    // ------------------------------------------------------- producer ----
    if (lane == 0) {
      const size_t a_tile0 = (size_t)mt * KS;
      const size_t b_tile0 = ((size_t)expert * NB + (size_t)nt * C::kHalves) * KS;
      // copy only the valid rows of the activation code tiles
      const uint32_t a_rows = (uint32_t)valid;
      const uint32_t a_trim = (128u - a_rows) * (sharq ? 208u : 128u);
      auto issue_b = [&](uint8_t* st, uint64_t* fb, size_t b_tile, int ks) {
#pragma unroll
        for (int h = 0; h < C::kHalves; ++h) {
          const size_t bt = b_tile + (size_t)h * KS + ks;
          bulk_g2s(st + C::kOffB + h * kCodesTile, args.w_codes + bt * kCodesTile, kCodesTile, fb);
          bulk_g2s(st + C::kOffSFB16 + h * kSf16Tile, args.w_sf16 + bt * kSf16Tile, kSf16Tile, fb);
          if (sharq) bulk_g2s(st + C::kOffSFB32 + h * kSf32Tile, args.w_sf32 + bt * kSf32Tile, kSf32Tile, fb);
        }
      };
      auto issue_a = [&](uint8_t* st, uint64_t* fb, size_t at) {
        bulk_g2s(st + C::kOffAR, args.a_r + at * kCodesTile, a_rows * 128u, fb);
        bulk_g2s(st + C::kOffSFAR, args.a_rsf + at * kSf16Tile, kSf16Tile, fb);
        if (sharq) {
          bulk_g2s(st + C::kOffASP, args.a_sp + at * kSpTile, a_rows * 64u, fb);
          bulk_g2s(st + C::kOffE, args.a_meta + at * kMetaTile, a_rows * 16u, fb);
          bulk_g2s(st + C::kOffSFASP, args.a_spsf + at * kSf32Tile, kSf32Tile, fb);
        }
      };
      if (kFused) {
        // weight half only; the A half is written by the epilogue warps
        for (int i = 0; i < nks; ++i) {
          const int s = i % C::kStages;
          if (i >= C::kStages) {
            if (!mbar_wait(&empty_bar[s], ((i / C::kStages) & 1) ^ 1, deadline, &abort_sh)) {
              record_error(args.err, kErrTimeout);
              abort_sh = 1;
              break;
            }
          }
          mbar_arrive_expect_tx(&full_bar[s], C::kTxB);
          issue_b(smem + s * C::kStageBytes, &full_bar[s], b_tile0, ks0 + i);
          if (i == 0) TRACE_POINT(2);
        }
      } else {
      // The weights do not depend on the preceding kernel (sharq_prep): issue
      // the weight copies of the first ring's worth of stages before waiting
      // for it (programmatic dependent launch), then the activation copies.
      const int pre = nks < C::kStages ? nks : C::kStages;
      for (int i = 0; i < pre; ++i) {
        uint8_t* st = smem + i * C::kStageBytes;
        mbar_arrive_expect_tx(&full_bar[i], (sharq ? C::kTxSharq : C::kTxNvfp4) - a_trim);
        issue_b(st, &full_bar[i], b_tile0, ks0 + i);
      }
      grid_dependency_wait();
      for (int i = 0; i < pre; ++i) issue_a(smem + i * C::kStageBytes, &full_bar[i], a_tile0 + ks0 + i);
      if (pre > 0) TRACE_POINT(2);
      if (blockIdx.x == 0 && blockIdx.z == 0 && args.act_err && *args.act_err) record_error(args.err, *args.act_err);
      for (int i = pre; i < nks; ++i) {
        const int s = i % C::kStages;
        if (!mbar_wait(&empty_bar[s], ((i / C::kStages) & 1) ^ 1, deadline, &abort_sh)) {
          record_error(args.err, kErrTimeout);
          abort_sh = 1;
          break;
        }
        uint8_t* st = smem + s * C::kStageBytes;
        mbar_arrive_expect_tx(&full_bar[s], (sharq ? C::kTxSharq : C::kTxNvfp4) - a_trim);
        issue_b(st, &full_bar[s], b_tile0, ks0 + i);
        issue_a(st, &full_bar[s], a_tile0 + ks0 + i);
      }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA ----
    if (lane == 0) {
      constexpr uint32_t idesc_dn = idesc_nvf4(128, BN, false);
      constexpr uint32_t idesc_sp = idesc_nvf4(128, BN, true);
      for (int i = 0; i < nks; ++i) {
        const int s = i % C::kStages;
        if (!mbar_wait(&full_bar[s], (i / C::kStages) & 1, deadline, &abort_sh)) {
          record_error(args.err, kErrTimeout);
          abort_sh = 1;
          break;
        }
        tc_fence_after();
        if (i == 0) TRACE_POINT(3);
        const uint32_t st = smem_u32(smem + s * C::kStageBytes);
        const uint32_t sf = tmem + C::kColSf0 + (uint32_t)s * C::kSfRegion;
        if (kFused) {  // the activation half, written by the epilogue warps
          if (!mbar_wait(&afull_bar[s], (i / C::kStages) & 1, deadline, &abort_sh)) {
            record_error(args.err, kErrTimeout);
            abort_sh = 1;
            break;
          }
        }
        // this stage's scale factors and metadata, copied by the copy warps
        if (!mbar_wait(&sf_full[s], (i / C::kStages) & 1, deadline, &abort_sh)) {
          record_error(args.err, kErrTimeout);
          abort_sh = 1;
          break;
        }
        tc_fence_after();
        if (sharq) {
          // sparse backbone: 2 x (128 x BN x 128 logical K)
#pragma unroll
          for (int j = 0; j < 2; ++j)
            mma_sp_nvf4(tmem + C::kColAcc, smem_desc(st + C::kOffASP + 32 * j, 16, 512, kSw64),
                        smem_desc(st + C::kOffB + 64 * j, 16, 1024, kSw128), sf + C::kSfE + 2 * j, idesc_sp,
                        sf + C::kSfASP + 4 * j, sf + C::kSfB32 + j * C::kSfbCols, (i > 0 || j > 0) ? 1u : 0u);
        }
        // dense residual: 4 x (128 x BN x 64 K), same accumulator, same B tile
#pragma unroll
        for (int j = 0; j < 4; ++j)
          mma_nvf4(tmem + C::kColAcc, smem_desc(st + C::kOffAR + 32 * j, 16, 1024, kSw128),
                   smem_desc(st + C::kOffB + 32 * j, 16, 1024, kSw128), idesc_dn, sf + C::kSfAR + 4 * j,
                   sf + C::kSfB16 + j * C::kSfbCols, (sharq || i > 0 || j > 0) ? 1u : 0u);
        tc_commit(&empty_bar[s]);
      }
      tc_commit(&acc_bar);  // accumulator complete (or everything issued so far, on abort)
      TRACE_POINT(4);
    }
  } else if (warp >= 6) {
    // ---------------------------------------------------- copy warps ----
    if (lane == 0) {
      const int cw = warp - 6;
      for (int i = 0; i < nks; ++i) {
        const int s = i % C::kStages;
        // the stage's data has landed (the slot, and with it its scale
        // region, is refilled only after the MMAs that read it completed)
        if (!mbar_wait(&full_bar[s], (i / C::kStages) & 1, deadline, &abort_sh)) {
          record_error(args.err, kErrTimeout);
          abort_sh = 1;
          break;
        }
        tc_fence_after();
        const uint32_t st = smem_u32(smem + s * C::kStageBytes);
        const uint32_t sf = tmem + C::kColSf0 + (uint32_t)s * C::kSfRegion;
        int n = 0;
        copies_weight<C>(st, sf, sharq, cw, n);
        if (kFused) {  // the activation half comes from the epilogue warps
          if (!mbar_wait(&afull_bar[s], (i / C::kStages) & 1, deadline, &abort_sh)) {
            record_error(args.err, kErrTimeout);
            abort_sh = 1;
            break;
          }
          tc_fence_after();
        }
        copies_act<C>(st, sf, sharq, cw, n);
        tc_commit(&sf_full[s]);
      }
      // every copy this warp issued has landed before the TMEM is freed
      tc_commit(&cp_fin[cw]);
      const uint64_t lim = globaltimer_ns() + kWaitLimitNs;
      while (!mbar_try_wait(&cp_fin[cw], 0) && globaltimer_ns() < lim) {
      }
    }
  } else {
    // ------------------------------------------------------- epilogue ----
    const int sp = warp & 3;  // TMEM lane quarter this warp may access
    const int rl = sp * 32 + lane;
    if (kFused && !fused_prep<C, kSplit>(args, smem, ks0, nks, valid, S, deadline, &abort_sh, empty_bar, afull_bar,
                                         stat_bar, fstats)) {
      record_error(args.err, kErrTimeout);
      abort_sh = 1;
    }
    const bool ok = mbar_wait(&acc_bar, 0, deadline, &abort_sh);
    tc_fence_after();
    grid_dependency_wait();  // s_g is written by the preceding sharq_prep
    if (threadIdx.x == 64) TRACE_POINT(5);
    if (!ok) {
      record_error(args.err, kErrTimeout);
      abort_sh = 1;
    } else if (!kSplit) {
      const int row = mt * 128 + rl;
      const float scale =
          __fmul_rn(kFused ? fstats.s : args.s_g[args.per_token ? row : 0], args.s_w[expert]);
#pragma unroll 1
      for (int c = 0; c < BN; c += 32) {
        uint32_t v[32];
        tmem_ld32(tmem + ((uint32_t)(sp * 32) << 16) + C::kColAcc + c, v);
        tmem_ld_wait();
        if (rl < valid) store_row32(args.Y, args.out_f32, (size_t)row * args.D + nt * BN + c, v, scale);
      }
    } else {
      // push this split's partial row straight from registers into the
      // owner CTA's receive buffer, laid out [sender][column quad][row of the
      // slice (+1 pad)][4 floats]: the lanes of a warp hold consecutive rows,
      // so each of their stores is one contiguous 512-byte run
      const int owner = rl / max(rows_per, 1);
      const int rp = rows_per + 1;  // padded: the owner's quad-major reads stay conflict-free
      const uint32_t dst =
          rl < valid ? mapa_shared(smem_u32(smem + C::kRingBytes) +
                                       (uint32_t)((split * (BN / 4) * rp + (rl - owner * rows_per)) * 16),
                                   (uint32_t)owner)
                     : 0u;
      const uint32_t rbar = rl < valid ? mapa_shared(smem_u32(&recv_bar), (uint32_t)owner) : 0u;
#pragma unroll 1
      for (int c = 0; c < BN; c += 32) {
        uint32_t v[32];
        tmem_ld32(tmem + ((uint32_t)(sp * 32) << 16) + C::kColAcc + c, v);
        tmem_ld_wait();
        if (rl < valid) {
#pragma unroll
          for (int q = 0; q < 32; q += 4)
            st_async_f4(dst + (uint32_t)((c + q) / 4 * rp) * 16u, __uint_as_float(v[q]), __uint_as_float(v[q + 1]),
                        __uint_as_float(v[q + 2]), __uint_as_float(v[q + 3]), rbar);
        }
      }
    }
  }

  if (threadIdx.x == 64) TRACE_POINT(6);
  if (kFused) __syncthreads();  // fstats.s visible to every warp
  if (kSplit && my_n > 0) {
    grid_dependency_wait();
    // ------------------------ owner: sum the S received slices in rank order
    bool ok = !abort_sh;
    while (ok && !mbar_try_wait_cluster(&recv_bar, 0)) {
      if (globaltimer_ns() > deadline) ok = false;
    }
    if (!ok) {
      if (threadIdx.x == 0) record_error(args.err, kErrTimeout);
    } else {
      const float sw = args.s_w[expert];
      const float* recv = reinterpret_cast<const float*>(smem + C::kRingBytes);
      constexpr int q4 = BN / 4;
      const int rp = rows_per + 1;
      for (int idx = threadIdx.x; idx < my_n * q4; idx += C::kThreadsT) {
        const int r = idx / q4, c4 = idx - r * q4;  // consecutive threads: consecutive columns of a row
        const float* p = recv + ((size_t)c4 * rp + r) * 4;
        float4 acc = *reinterpret_cast<const float4*>(p);
        for (int s2 = 1; s2 < S; ++s2) {
          const float4 q = *reinterpret_cast<const float4*>(p + (size_t)s2 * q4 * rp * 4);
          acc.x = __fadd_rn(acc.x, q.x);
          acc.y = __fadd_rn(acc.y, q.y);
          acc.z = __fadd_rn(acc.z, q.z);
          acc.w = __fadd_rn(acc.w, q.w);
        }
        const int row = mt * 128 + my0 + r;
        const float scale = __fmul_rn(kFused ? fstats.s : args.s_g[args.per_token ? row : 0], sw);
        store4(args.Y, args.out_f32, (size_t)row * args.D + nt * BN + 4 * c4, acc, scale);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0) TRACE_POINT(7);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// Persistent form (no split-K, activation already prepared: prefill, the
// grouped expert shapes, and every shape of the Table-5 operand modes).  One
// CTA per SM walks the output tiles t = blockIdx.x, blockIdx.x + gridDim.x,
// ... (row-major over (m-tile, n-tile), so CTAs running at the same time
// share activation tiles in L2).  The shared-memory ring and its phases run on
// across tiles, so the producer streams the next tile's stages while the
// current one finishes, and the accumulator is handed back to the MMA warp as
// soon as the epilogue has moved it into registers (bf16 output: the tile's
// row in 128 packed registers per thread) -- the global stores of tile k
// overlap the MMAs of tile k + 1.  Set-up (barriers, TMEM allocation) is paid
// once per SM.
//
// Operand sets (kG): both FP4 operands of the activation accumulate into one
// TMEM tile and read the same weight tile; a sparse operand (4:8 in-pairs,
// one scale per 32 logical K) pairs with the weight's per-32 scale view, a
// dense one (one scale per 16 K) with the per-16 view.
enum : int {
  kGemmSharq = 0, kGemmNvfp4 = 1, kGemmSparseOnly = 2, kGemmDenseDense = 3, kGemmSparseSparse = 4,
  kGemmSharqMx = 5,  // MXFP4 operands (kind::mxf4, E8M0): sparse backbone + dense residual
  kGemmMxfp4 = 6     // plain MXFP4: one dense operand
};

template <int BN, int kG>
struct PCfg {
  static constexpr int kHalves = BN / 128;
  // copy warps: 4 for 128-wide tiles; 2 for 256-wide ones, whose epilogue
  // keeps a 256-column row in registers (65536 / 256 threads per thread)
  static constexpr int kCW = BN == 256 ? 2 : 4;
  static constexpr int kThreadsT = gemm_threads(kCW);
  static constexpr bool kMx = kG == kGemmSharqMx || kG == kGemmMxfp4;
  static constexpr bool kHas1 = kG != kGemmNvfp4 && kG != kGemmMxfp4;  // first operand (backbone)
  static constexpr bool kSp1 = kG != kGemmDenseDense;                 // ... sparse
  static constexpr bool kHas2 = kG != kGemmSparseOnly;                // second operand (residual)
  static constexpr bool kSp2 = kG == kGemmSparseSparse;
  static constexpr bool kB32 = (kHas1 && kSp1) || (kHas2 && kSp2);    // weight sparse-path view
  static constexpr bool kB16 = (kHas1 && !kSp1) || (kHas2 && !kSp2);  // weight dense-path view
  // scale tiles: NVFP4 sparse 1 KB (per 32 logical K), dense 2 KB (per 16);
  // MXFP4 sparse 512 B (per 64 logical K), dense 1 KB (per 32)
  static constexpr int kSfSp = kMx ? kSf64Tile : kSf32Tile;
  static constexpr int kSfDn = kMx ? kSf32Tile : kSf16Tile;
  static constexpr int kA1 = kHas1 ? (kSp1 ? kSpTile : kCodesTile) : 0;
  static constexpr int kE1 = kHas1 && kSp1 ? kMetaTile : 0;
  static constexpr int kS1 = kHas1 ? (kSp1 ? kSfSp : kSfDn) : 0;
  static constexpr int kA2 = kHas2 ? (kSp2 ? kSpTile : kCodesTile) : 0;
  static constexpr int kE2 = kHas2 && kSp2 ? kMetaTile : 0;
  static constexpr int kS2 = kHas2 ? (kSp2 ? kSfSp : kSfDn) : 0;
  // stage layout: the swizzled code tiles first (1 KB multiples), then
  // metadata and scales
  static constexpr int kOffB = 0;
  static constexpr int kOffA2 = kOffB + BN * 128;
  static constexpr int kOffA1 = kOffA2 + kA2;
  static constexpr int kOffE1 = kOffA1 + kA1;
  static constexpr int kOffE2 = kOffE1 + kE1;
  static constexpr int kOffS1 = kOffE2 + kE2;
  static constexpr int kOffS2 = kOffS1 + kS1;
  static constexpr int kOffSFB32 = kOffS2 + kS2;
  static constexpr int kOffSFB16 = kOffSFB32 + (kB32 ? kHalves * kSfSp : 0);
  // rounded to 1 KB so that every stage's swizzled code tiles (first in the
  // stage) stay 1024-byte aligned; the scale regions need only 16 bytes
  static constexpr int kStageBytes = (kOffSFB16 + (kB16 ? kHalves * kSfDn : 0) + 1023) / 1024 * 1024;
  static constexpr int kStages = (BN == 128 && 4 * kStageBytes + 4 * 4096 + 1024 <= 232448) ? 4 : 3;
  // bf16 output staging after the ring, 4 KB per epilogue warp, where it fits
  // (not beside the three 72 KB stages of the Dense+Dense operand set)
  static constexpr bool kStaged = kStages * kStageBytes + 4 * 4096 + 1024 <= 232448;
  static constexpr int kOffStage = kStages * kStageBytes;
  static constexpr int kSmemBytes = kOffStage + (kStaged ? 4 * 4096 : 0) + 1024;
  // TMEM: accumulator, then one scale region per ring slot: 32 activation
  // columns + the weight scale columns
  static constexpr uint32_t kColAcc = 0;
  static constexpr uint32_t kSfbCols = BN / 32;
  static constexpr uint32_t kSfE1 = 0, kSfE2 = 4, kSfS1 = kSp1 ? 8 : 0, kSfS2 = 16;
  static constexpr uint32_t kSfB32 = 32, kSfB16 = 32 + 2 * kSfbCols;
  static constexpr uint32_t kSfRegion = 32 + 6 * kSfbCols;
  static constexpr uint32_t kColSf0 = BN;
  static constexpr uint32_t kTmemCols = BN + kStages * kSfRegion <= 256 ? 256 : 512;
  // transaction bytes per stage with `rows` valid activation rows
  __host__ __device__ static constexpr uint32_t tx(uint32_t rows) {
    return BN * 128 + (kB32 ? kHalves * kSfSp : 0) + (kB16 ? kHalves * kSfDn : 0) +
           rows * (uint32_t)(kA1 / 128 + kE1 / 128 + kA2 / 128 + kE2 / 128) + kS1 + kS2;
  }
  static_assert(kStageBytes % 1024 == 0, "stage must keep 1024-byte alignment");
  static_assert(kSmemBytes <= 232448, "shared memory overflow");
  static_assert(BN + kStages * kSfRegion <= 512, "TMEM overflow");
};

// The scale-factor and metadata copies of one stage of the persistent
// kernel (shared memory -> TMEM scale region sf): the weight views the
// operand set needs, then each activation operand's metadata and scales.
// Copy number n is issued by copy warp n % kCW.
template <class C>
__device__ __forceinline__ void stage_copies(uint32_t st, uint32_t sf, int cw) {
  int n = 0;
  auto cp4 = [&](uint32_t taddr, uint32_t saddr) {
    if (n++ % C::kCW == cw) tc_cp_32x128b_x4(taddr, smem_desc(saddr, 0, 128, kSwNone));
  };
  auto cpm = [&](uint32_t taddr, uint32_t saddr) {
    if (n++ % C::kCW == cw) tc_cp_128x128b(taddr, smem_desc(saddr, 0, 128, kSwNone));
  };
  // atoms (512 B, 4 TMEM columns) per 256-K stage: NVFP4 sparse 2 / dense 4,
  // MXFP4 sparse 1 / dense 2
  constexpr int kAtSp = C::kMx ? 1 : 2, kAtDn = C::kMx ? 2 : 4;
  if (C::kB32) {
#pragma unroll
    for (int j = 0; j < kAtSp; ++j)
#pragma unroll
      for (int h = 0; h < C::kHalves; ++h)
        cp4(sf + C::kSfB32 + j * C::kSfbCols + 4 * h, st + C::kOffSFB32 + h * C::kSfSp + 512 * j);
  }
  if (C::kB16) {
#pragma unroll
    for (int j = 0; j < kAtDn; ++j)
#pragma unroll
      for (int h = 0; h < C::kHalves; ++h)
        cp4(sf + C::kSfB16 + j * C::kSfbCols + 4 * h, st + C::kOffSFB16 + h * C::kSfDn + 512 * j);
  }
  if (C::kHas1) {
    if (C::kSp1) cpm(sf + C::kSfE1, st + C::kOffE1);
#pragma unroll
    for (int j = 0; j < (C::kSp1 ? kAtSp : kAtDn); ++j) cp4(sf + C::kSfS1 + 4 * j, st + C::kOffS1 + 512 * j);
  }
  if (C::kHas2) {
    if (C::kSp2) cpm(sf + C::kSfE2, st + C::kOffE2);
#pragma unroll
    for (int j = 0; j < (C::kSp2 ? kAtSp : kAtDn); ++j) cp4(sf + C::kSfS2 + 4 * j, st + C::kOffS2 + 512 * j);
  }
}

template <int BN, int kG>
__global__ void __launch_bounds__(PCfg<BN, kG>::kThreadsT, 1)
    sharq_gemm_persistent_kernel(const GemmArgs args, int m_tiles) {
  using C = PCfg<BN, kG>;
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full_bar[C::kStages];
  __shared__ __align__(8) uint64_t empty_bar[C::kStages];
  __shared__ __align__(8) uint64_t acc_full;
  __shared__ __align__(8) uint64_t acc_empty;
  __shared__ __align__(8) uint64_t sf_full[C::kStages];  // ring slot s: its stage's copies have landed
  __shared__ __align__(8) uint64_t cp_fin[C::kCW];  // each copy warp's last copies
  __shared__ uint32_t tmem_base_sh;
  __shared__ volatile int abort_sh;

  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int KS = args.K >> 8;
  const int NB = args.D >> 7;
  const int n_tiles = args.D / BN;
  const int ntiles = m_tiles * n_tiles;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    mbar_init(&acc_full, 1);
    mbar_init(&acc_empty, 4);  // each epilogue warp, once per tile
    for (int st = 0; st < C::kStages; ++st) mbar_init(&sf_full[st], C::kCW);
    for (int c = 0; c < C::kCW; ++c) mbar_init(&cp_fin[c], 1);
    fence_mbar_init();
    abort_sh = 0;
  }
  if (warp == 1) {
    tmem_alloc(&tmem_base_sh, C::kTmemCols);
    tmem_relinquish();
  }
  if (C::kE1 || C::kE2) {
    // Metadata rows past a partial tile's valid rows are never copied in: give
    // every row a valid pattern (pairs 0 and 1) once; later tiles leave
    // metadata written by sharq_prep there, which is valid as well.
    for (int idx = threadIdx.x; idx < C::kStages * 128; idx += C::kThreadsT) {
      const int st = idx >> 7, row = idx & 127;
      const uint4 v = make_uint4(0x44444444u, 0x44444444u, 0x44444444u, 0x44444444u);
      if (C::kE1) *reinterpret_cast<uint4*>(smem + st * C::kStageBytes + C::kOffE1 + row * 16) = v;
      if (C::kE2) *reinterpret_cast<uint4*>(smem + st * C::kStageBytes + C::kOffE2 + row * 16) = v;
    }
    fence_proxy_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;

  if (warp == 0) {
    // ------------------------------------------------------- producer ----
    if (lane == 0) {
      grid_dependency_wait();  // the activation comes from the preceding sharq_prep
      if (blockIdx.x == 0 && args.act_err && *args.act_err) record_error(args.err, *args.act_err);
      uint32_t g = 0;  // stage counter across tiles
      for (int tile = blockIdx.x; tile < ntiles && !abort_sh; tile += gridDim.x) {
        int mt, nt;
        tile_coords(tile, m_tiles, n_tiles, args.n_major, mt, nt);
        const int expert = tile_expert(args, mt);
        if (expert < 0) {
          if (nt == 0) record_error(args.err, kErrInvalid);
          continue;
        }
        const uint64_t deadline = globaltimer_ns() + kWaitLimitNs;
        const uint32_t rows = (uint32_t)min(128, args.T - mt * 128);
        const uint32_t tx = C::tx(rows);
        const size_t a_tile0 = (size_t)mt * KS;
        const size_t b_tile0 = ((size_t)expert * NB + (size_t)nt * C::kHalves) * KS;
        for (int i = 0; i < KS; ++i, ++g) {
          const int s = g % C::kStages;
          if (g >= (uint32_t)C::kStages &&
              !mbar_wait(&empty_bar[s], ((g / C::kStages) & 1) ^ 1, deadline, &abort_sh)) {
            record_error(args.err, kErrTimeout);
            abort_sh = 1;
            break;
          }
          uint8_t* st = smem + s * C::kStageBytes;
          uint64_t* fb = &full_bar[s];
          mbar_arrive_expect_tx(fb, tx);
#pragma unroll
          for (int h = 0; h < C::kHalves; ++h) {
            const size_t bt = b_tile0 + (size_t)h * KS + i;
            bulk_g2s(st + C::kOffB + h * kCodesTile, args.w_codes + bt * kCodesTile, kCodesTile, fb);
            if (C::kB16) bulk_g2s(st + C::kOffSFB16 + h * C::kSfDn, args.w_sf16 + bt * C::kSfDn, C::kSfDn, fb);
            if (C::kB32) bulk_g2s(st + C::kOffSFB32 + h * C::kSfSp, args.w_sf32 + bt * C::kSfSp, C::kSfSp, fb);
          }
          const size_t at = a_tile0 + i;
          if (C::kHas1) {
            bulk_g2s(st + C::kOffA1, args.a_sp + at * C::kA1, rows * (C::kA1 / 128), fb);
            if (C::kE1) bulk_g2s(st + C::kOffE1, args.a_meta + at * kMetaTile, rows * 16u, fb);
            bulk_g2s(st + C::kOffS1, args.a_spsf + at * C::kS1, C::kS1, fb);
          }
          if (C::kHas2) {
            bulk_g2s(st + C::kOffA2, args.a_r + at * C::kA2, rows * (C::kA2 / 128), fb);
            if (C::kE2) bulk_g2s(st + C::kOffE2, args.a_rmeta + at * kMetaTile, rows * 16u, fb);
            bulk_g2s(st + C::kOffS2, args.a_rsf + at * C::kS2, C::kS2, fb);
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA ----
    if (lane == 0) {
      constexpr uint32_t idesc_dn = idesc_nvf4(128, BN, false);
      constexpr uint32_t idesc_sp = idesc_nvf4(128, BN, true);
      uint32_t g = 0, k = 0;  // stage counter, tiles done
      for (int tile = blockIdx.x; tile < ntiles && !abort_sh; tile += gridDim.x) {
        int tmt, tnt;
        tile_coords(tile, m_tiles, n_tiles, args.n_major, tmt, tnt);
        if (tile_expert(args, tmt) < 0) continue;
        const uint64_t deadline = globaltimer_ns() + kWaitLimitNs;
        // the epilogue has taken the previous tile's accumulator
        if (k > 0 && !mbar_wait(&acc_empty, (k - 1) & 1, deadline, &abort_sh)) {
          record_error(args.err, kErrTimeout);
          abort_sh = 1;
          break;
        }
        tc_fence_after();
        for (int i = 0; i < KS; ++i, ++g) {
          const int s = g % C::kStages;
          if (!mbar_wait(&full_bar[s], (g / C::kStages) & 1, deadline, &abort_sh)) {
            record_error(args.err, kErrTimeout);
            abort_sh = 1;
            break;
          }
          tc_fence_after();
          // this stage's scale factors and metadata, copied by the copy warps
          if (!mbar_wait(&sf_full[s], (g / C::kStages) & 1, deadline, &abort_sh)) {
            record_error(args.err, kErrTimeout);
            abort_sh = 1;
            break;
          }
          tc_fence_after();
          const uint32_t st = smem_u32(smem + s * C::kStageBytes);
          const uint32_t sf = tmem + C::kColSf0 + (uint32_t)s * C::kSfRegion;
          bool acc = i > 0;  // the tile's first MMA overwrites the accumulator
          // a sparse operand: 2 x (128 x BN x 128 logical K), weight per-32 view
          auto sparse_op = [&](uint32_t a_off, uint32_t e_col, uint32_t s_col) {
#pragma unroll
            for (int j = 0; j < 2; ++j) {
              mma_sp_nvf4(tmem + C::kColAcc, smem_desc(st + a_off + 32 * j, 16, 512, kSw64),
                          smem_desc(st + C::kOffB + 64 * j, 16, 1024, kSw128), sf + e_col + 2 * j, idesc_sp,
                          sf + s_col + 4 * j, sf + C::kSfB32 + j * C::kSfbCols, acc ? 1u : 0u);
              acc = true;
            }
          };
          // a dense operand: 4 x (128 x BN x 64 K), weight per-16 view
          auto dense_op = [&](uint32_t a_off, uint32_t s_col) {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              mma_nvf4(tmem + C::kColAcc, smem_desc(st + a_off + 32 * j, 16, 1024, kSw128),
                       smem_desc(st + C::kOffB + 32 * j, 16, 1024, kSw128), idesc_dn, sf + s_col + 4 * j,
                       sf + C::kSfB16 + j * C::kSfbCols, acc ? 1u : 0u);
              acc = true;
            }
          };
          // MXFP4 (kind::mxf4, E8M0): one 512-byte atom holds 4 scales per row
          // = two MMAs' worth; the scale-factor ID (byte 0 or 2 of the
          // column) picks this MMA's pair, in the descriptor and in bits
          // 30-31 of the TMEM scale address
          auto sparse_op_mx = [&](uint32_t a_off, uint32_t e_col, uint32_t s_col) {
#pragma unroll
            for (int j = 0; j < 2; ++j) {
              const uint32_t id = 2u * j;
              mma_sp_mxf4(tmem + C::kColAcc, smem_desc(st + a_off + 32 * j, 16, 512, kSw64),
                          smem_desc(st + C::kOffB + 64 * j, 16, 1024, kSw128), sf + e_col + 2 * j,
                          idesc_mxf4(128, BN, true, id, id), (sf + s_col) | (id << 30),
                          (sf + C::kSfB32) | (id << 30), acc ? 1u : 0u);
              acc = true;
            }
          };
          auto dense_op_mx = [&](uint32_t a_off, uint32_t s_col) {
#pragma unroll
            for (int a = 0; a < 2; ++a) {
#pragma unroll
              for (int q = 0; q < 2; ++q) {
                const int j = 2 * a + q;
                const uint32_t id = 2u * q;
                mma_mxf4(tmem + C::kColAcc, smem_desc(st + a_off + 32 * j, 16, 1024, kSw128),
                         smem_desc(st + C::kOffB + 32 * j, 16, 1024, kSw128), idesc_mxf4(128, BN, false, id, id),
                         (sf + s_col + 4 * a) | (id << 30), (sf + C::kSfB16 + a * C::kSfbCols) | (id << 30),
                         acc ? 1u : 0u);
                acc = true;
              }
            }
          };
          if (C::kMx) {
            if (C::kHas1) sparse_op_mx(C::kOffA1, C::kSfE1, C::kSfS1);
            dense_op_mx(C::kOffA2, C::kSfS2);
          } else {
            if (C::kHas1) {
              if (C::kSp1) sparse_op(C::kOffA1, C::kSfE1, C::kSfS1);
              else dense_op(C::kOffA1, C::kSfS1);
            }
            if (C::kHas2) {
              if (C::kSp2) sparse_op(C::kOffA2, C::kSfE2, C::kSfS2);
              else dense_op(C::kOffA2, C::kSfS2);
            }
          }
          tc_commit(&empty_bar[s]);
        }
        tc_commit(&acc_full);  // accumulator of this tile complete
        ++k;
      }
    }
  } else if (warp >= 6) {
    // ---------------------------------------------------- copy warps ----
    if (lane == 0) {
      const int cw = warp - 6;
      uint32_t g = 0;  // stage counter across tiles, as the MMA warp's
      for (int tile = blockIdx.x; tile < ntiles && !abort_sh; tile += gridDim.x) {
        int tmt, tnt;
        tile_coords(tile, m_tiles, n_tiles, args.n_major, tmt, tnt);
        if (tile_expert(args, tmt) < 0) continue;
        const uint64_t deadline = globaltimer_ns() + kWaitLimitNs;
        for (int i = 0; i < KS; ++i, ++g) {
          const int s = g % C::kStages;
          // the stage's data has landed (the slot, and with it its scale
          // region, is refilled only after the MMAs that read it completed)
          if (!mbar_wait(&full_bar[s], (g / C::kStages) & 1, deadline, &abort_sh)) {
            record_error(args.err, kErrTimeout);
            abort_sh = 1;
            break;
          }
          tc_fence_after();
          stage_copies<C>(smem_u32(smem + s * C::kStageBytes), tmem + C::kColSf0 + (uint32_t)s * C::kSfRegion, cw);
          tc_commit(&sf_full[s]);
        }
      }
      // every copy this warp issued has landed before the TMEM is freed
      tc_commit(&cp_fin[cw]);
      const uint64_t lim = globaltimer_ns() + kWaitLimitNs;
      while (!mbar_try_wait(&cp_fin[cw], 0) && globaltimer_ns() < lim) {
      }
    }
  } else {
    // ------------------------------------------------------- epilogue ----
    const int sp = warp & 3;  // TMEM lane quarter this warp may access
    const int rl = sp * 32 + lane;
    grid_dependency_wait();  // s_g is written by the preceding sharq_prep
    const float s_tensor = args.per_token ? 0.0f : *args.s_g;
    uint32_t k = 0;
    for (int tile = blockIdx.x; tile < ntiles && !abort_sh; tile += gridDim.x) {
      int mt, nt;
      tile_coords(tile, m_tiles, n_tiles, args.n_major, mt, nt);
      const int expert = tile_expert(args, mt);
      if (expert < 0) continue;
      const uint64_t deadline = globaltimer_ns() + kWaitLimitNs;
      if (!mbar_wait(&acc_full, k & 1, deadline, &abort_sh)) {
        record_error(args.err, kErrTimeout);
        abort_sh = 1;
        break;
      }
      tc_fence_after();
      const float scale =
          __fmul_rn(args.per_token ? args.s_g[mt * 128 + rl] : s_tensor, args.s_w[expert]);
      const int valid = min(128, args.T - mt * 128);
      const size_t off = (size_t)(mt * 128 + rl) * args.D + (size_t)nt * BN;
      if (!args.out_f32) {
        uint32_t pk[BN / 2];  // the row as packed bf16, then the accumulator is free
#pragma unroll
        for (int c = 0; c < BN; c += 32) {
          uint32_t v[32];
          tmem_ld32(tmem + ((uint32_t)(sp * 32) << 16) + C::kColAcc + c, v);
          tmem_ld_wait();
#pragma unroll
          for (int q = 0; q < 16; ++q) {
            __nv_bfloat162 b2 = __floats2bfloat162_rn(__fmul_rn(__uint_as_float(v[2 * q]), scale),
                                                      __fmul_rn(__uint_as_float(v[2 * q + 1]), scale));
            pk[c / 2 + q] = *reinterpret_cast<uint32_t*>(&b2);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_local(&acc_empty);  // the warp's rows are in registers
        if constexpr (C::kStaged) {
          store_rows_bf16_staged<BN>(pk, smem + C::kOffStage + (size_t)sp * 4096,
                                     static_cast<__nv_bfloat16*>(args.Y) + (size_t)(mt * 128 + sp * 32) * args.D +
                                         (size_t)nt * BN,
                                     (size_t)args.D, valid - sp * 32, lane);
        } else if (rl < valid) {
          uint4* y = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(args.Y) + off);
#pragma unroll
          for (int q = 0; q < BN / 8; ++q) y[q] = make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
        }
      } else {
#pragma unroll 1
        for (int c = 0; c < BN; c += 32) {
          uint32_t v[32];
          tmem_ld32(tmem + ((uint32_t)(sp * 32) << 16) + C::kColAcc + c, v);
          tmem_ld_wait();
          if (rl < valid) store_row32(args.Y, 1, off + c, v, scale);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_local(&acc_empty);
      }
      ++k;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// Pair form (prefill): two CTAs of a cluster run each 256 x 256 output tile
// as one tensor-core unit (tcgen05 cta_group::2, M = 256).  CTA r of the pair
// holds the tile's rows 128 r .. 128 r + 127 of the activation operands and
// weight rows (output columns) 128 r .. 128 r + 127 of the shared FP4 weight
// payload; the MMA reads B from both CTAs' shared memory, so each weight byte
// crosses from L2 once per 256 activation rows instead of once per 128.  Per
// CTA and 256-K stage that is 51 KB of operands (backbone, metadata, residual,
// their scales, half the weight codes and both weight scale views) against
// 67 KB in the one-CTA form, for the same tensor-core work.
//   both CTAs  producer (warp 0): its own operand copies into its own ring of
//              four stages;
//              epilogue (warps 4-7): its own 128 accumulator rows.
//   even CTA   MMA issuer (warp 1): both operands' MMAs with cta_group::2,
//              committed to the ring slots of both CTAs at once (multicast)
//              and to the stage's TMEM scale region;
//              copy warps (2-3, 8-15): the stage's 19 scale and metadata
//              copies into both CTAs' TMEM (each from its own shared memory)
//              with cta_group::2.  Measured on B200 beside the MMAs, one warp
//              issues a copy every ~75 ns, so a stage's copies keep pace with
//              its six MMAs (~440 ns) only when spread over ten warps.
//   odd CTA    warp 1 forwards "stage landed" to the even CTA: plain bulk
//              copies complete only their own CTA's barrier, so it waits on
//              its barrier and arrives on the even CTA's.
// TMEM holds the 256-column accumulator and three scale regions (80 columns
// each), so the shared-memory ring (four slots) runs one stage deeper than
// the regions: the copies of stage g go to region g % 3 once the MMAs of
// stage g - 3 have completed.  Both CTAs' epilogue threads release the
// accumulator on the even CTA's barrier once the tile is in registers, before
// their global stores, so the stores overlap the next tile's MMAs.  The
// epilogue warpgroup takes 224 registers per thread (setmaxnreg), the other
// three give theirs down to 96 (4 x 128 threads x their shares = the launch's
// 65536).  Used for ungrouped SharQ and plain-NVFP4
// GEMMs with at least two 128-row tiles; a pair's second m-tile may lie past
// the activation's end (an odd tile count), in which case that CTA copies no
// activation bytes and stores nothing.
template <int kG>
struct PairCfg {
  static constexpr bool kHas1 = kG == kGemmSharq;  // the sparse backbone operand
  static constexpr int BN = 256;                   // output columns per tile (both CTAs)
  static constexpr int kWarps = 16;
  static constexpr int kThreadsT = 32 * kWarps;
  static constexpr int kCW = 10;                   // copy warps: 2, 3, 8..15
  static constexpr int kEpiWarp0 = 4;              // epilogue warps 4..7 (TMEM lane quarters 0..3)
  static constexpr int kRegsEpi = 224, kRegsOther = 96;  // setmaxnreg shares (x 128 threads each)
  static constexpr int kOffB = 0;                         // this CTA's 128 weight rows
  static constexpr int kOffA2 = kOffB + kCodesTile;       // residual (NVFP4: Xn) codes
  static constexpr int kOffA1 = kOffA2 + kCodesTile;      // backbone codes
  static constexpr int kOffE1 = kOffA1 + (kHas1 ? kSpTile : 0);
  static constexpr int kOffS1 = kOffE1 + (kHas1 ? kMetaTile : 0);
  static constexpr int kOffS2 = kOffS1 + (kHas1 ? kSf32Tile : 0);
  static constexpr int kOffSFB32 = kOffS2 + kSf16Tile;    // both weight halves' views
  static constexpr int kOffSFB16 = kOffSFB32 + (kHas1 ? 2 * kSf32Tile : 0);
  static constexpr int kStageBytes = (kOffSFB16 + 2 * kSf16Tile + 1023) / 1024 * 1024;
  static constexpr int kStages = 4;  // shared-memory ring slots
  static constexpr int kRegions = 3;  // TMEM scale regions
  // TMEM: the 256-column accumulator and the scale regions
  static constexpr uint32_t kSfbCols = BN / 32;
  static constexpr uint32_t kSfE1 = 0, kSfS1 = 8, kSfS2 = 16, kSfB32 = 32, kSfB16 = 32 + 2 * kSfbCols;
  static constexpr uint32_t kSfRegion = 32 + 6 * kSfbCols;
  static constexpr uint32_t kColAcc = 0, kColSf0 = BN;
  static constexpr uint32_t kTmemCols = 512;
  // bf16 output staging: 4 KB per epilogue warp (32 rows x 64 columns)
  static constexpr int kOffStage = kStages * kStageBytes;
  static constexpr int kSmemBytes = kOffStage + 4 * 4096 + 1024;
  // transaction bytes of one CTA's stage with `rows` valid activation rows
  __host__ __device__ static constexpr uint32_t tx(uint32_t rows) {
    return kCodesTile + (kHas1 ? 2 * kSf32Tile : 0) + 2 * kSf16Tile +
           (rows ? rows * (128u + (kHas1 ? 64u + 16u : 0u)) + (kHas1 ? kSf32Tile : 0) + kSf16Tile : 0u);
  }
  static_assert(kStageBytes % 1024 == 0, "stage must keep 1024-byte alignment");
  static_assert(kSmemBytes <= 232448, "shared memory overflow");
  static_assert(BN + kRegions * kSfRegion <= kTmemCols, "TMEM overflow");
  static_assert(kRegsEpi + 3 * kRegsOther <= 65536 / kThreadsT * 4, "register split above the launch's share");
};

// the pair kernel's register split (per thread; each warpgroup executes one)
__device__ __forceinline__ void regs_inc_epi() { asm volatile("setmaxnreg.inc.sync.aligned.u32 224;" ::: "memory"); }
__device__ __forceinline__ void regs_dec_other() { asm volatile("setmaxnreg.dec.sync.aligned.u32 96;" ::: "memory"); }

template <int kG>
__global__ void __launch_bounds__(PairCfg<kG>::kThreadsT, 1)
    sharq_gemm_pair_kernel(const GemmArgs args, int m_tiles) {
  using C = PairCfg<kG>;
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full_bar[C::kStages];
  __shared__ __align__(8) uint64_t empty_bar[C::kStages];
  __shared__ __align__(8) uint64_t peer_full[C::kStages];     // even CTA: the odd CTA's stage has landed
  __shared__ __align__(8) uint64_t sf_full[C::kRegions];      // even CTA: a region's copies have landed
  __shared__ __align__(8) uint64_t region_free[C::kRegions];  // even CTA: the MMAs reading a region are done
  __shared__ __align__(8) uint64_t acc_full;
  __shared__ __align__(8) uint64_t acc_empty;                 // even CTA: both epilogues took the accumulator
  __shared__ __align__(8) uint64_t cp_fin[C::kCW];
  __shared__ uint32_t tmem_base_sh;
  __shared__ volatile int abort_sh;

  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  const int KS = args.K >> 8;
  const int n_tiles = args.D / C::BN;
  const int m2_tiles = (m_tiles + 1) >> 1;
  const int ntiles = m2_tiles * n_tiles;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
      mbar_init(&peer_full[s], 1);
    }
    for (int r = 0; r < C::kRegions; ++r) {
      mbar_init(&sf_full[r], C::kCW);
      mbar_init(&region_free[r], 1);
    }
    mbar_init(&acc_full, 1);
    mbar_init(&acc_empty, 8);  // the 4 epilogue warps of each CTA, once per tile
    for (int c = 0; c < C::kCW; ++c) mbar_init(&cp_fin[c], 1);
    fence_mbar_init();
    abort_sh = 0;
  }
  if (warp == 1) {
    tmem_alloc_pair(&tmem_base_sh, C::kTmemCols);
    tmem_relinquish_pair();
  }
  if (C::kHas1) {
    // metadata of rows past a tile's valid rows is never copied in: a valid
    // pattern (pairs 0 and 1) everywhere once; later tiles leave metadata
    // written by sharq_prep there, which is valid as well
    for (int idx = threadIdx.x; idx < C::kStages * 128; idx += C::kThreadsT) {
      const int st = idx >> 7, row = idx & 127;
      *reinterpret_cast<uint4*>(smem + st * C::kStageBytes + C::kOffE1 + row * 16) =
          make_uint4(0x44444444u, 0x44444444u, 0x44444444u, 0x44444444u);
    }
    fence_proxy_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // the peer's barriers and TMEM exist before any pair traffic
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  const uint32_t peer_full_lead = mapa_shared(smem_u32(&peer_full[0]), 0);
  const uint32_t acc_empty_lead = mapa_shared(smem_u32(&acc_empty), 0);
  const int cw = warp == 2 || warp == 3 ? warp - 2 : (warp >= 8 ? warp - 6 : -1);  // copy warp index
  const bool epi_wg = warp >= C::kEpiWarp0 && warp < C::kEpiWarp0 + 4;

  if (!epi_wg) {
  regs_dec_other();  // warpgroups 0, 2 and 3 give registers to the epilogue
  if (warp == 0) {
    // ------------------------------------------------- producer (both) ----
    if (lane == 0) {
      grid_dependency_wait();  // the activation comes from the preceding sharq_prep
      if (blockIdx.x == 0 && args.act_err && *args.act_err) record_error(args.err, *args.act_err);
      uint32_t g = 0;
      for (int tile = pair; tile < ntiles && !abort_sh; tile += npairs) {
        int m2, nt;
        tile_coords(tile, m2_tiles, n_tiles, args.n_major, m2, nt);
        const int mt = 2 * m2 + (int)rank;
        const uint32_t rows = (uint32_t)max(0, min(128, args.T - mt * 128));
        const uint32_t tx = C::tx(rows);
        const uint64_t deadline = globaltimer_ns() + kWaitLimitNs;
        const size_t a_tile0 = (size_t)mt * KS;
        const size_t b_tile0 = (size_t)nt * 2 * KS;  // this column tile's first weight half
        for (int i = 0; i < KS; ++i, ++g) {
          const int s = g % C::kStages;
          if (g >= (uint32_t)C::kStages &&
              !mbar_wait(&empty_bar[s], ((g / C::kStages) & 1) ^ 1, deadline, &abort_sh)) {
            record_error(args.err, kErrTimeout);
            abort_sh = 1;
            break;
          }
          uint8_t* st = smem + s * C::kStageBytes;
          uint64_t* fb = &full_bar[s];
          mbar_arrive_expect_tx(fb, tx);
          // scales first: the copy warps need only those
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const size_t bh = b_tile0 + (size_t)h * KS + i;
            bulk_g2s(st + C::kOffSFB16 + h * kSf16Tile, args.w_sf16 + bh * kSf16Tile, kSf16Tile, fb);
            if (C::kHas1) bulk_g2s(st + C::kOffSFB32 + h * kSf32Tile, args.w_sf32 + bh * kSf32Tile, kSf32Tile, fb);
          }
          const size_t at = a_tile0 + i;
          if (rows) {
            bulk_g2s(st + C::kOffS2, args.a_rsf + at * kSf16Tile, kSf16Tile, fb);
            if (C::kHas1) {
              bulk_g2s(st + C::kOffE1, args.a_meta + at * kMetaTile, rows * 16u, fb);
              bulk_g2s(st + C::kOffS1, args.a_spsf + at * kSf32Tile, kSf32Tile, fb);
            }
          }
          const size_t bt = b_tile0 + (size_t)rank * KS + i;
          bulk_g2s(st + C::kOffB, args.w_codes + bt * kCodesTile, kCodesTile, fb);
          if (rows) {
            bulk_g2s(st + C::kOffA2, args.a_r + at * kCodesTile, rows * 128u, fb);
            if (C::kHas1) bulk_g2s(st + C::kOffA1, args.a_sp + at * kSpTile, rows * 64u, fb);
          }
        }
      }
      // every slot's last use has been released by the MMAs (their
      // completion arrives on this CTA's barriers) before the CTA may leave
      const uint64_t deadline = globaltimer_ns() + kWaitLimitNs;
      for (int j = 0; j < C::kStages && !abort_sh; ++j, ++g)
        if (g >= (uint32_t)C::kStages && !mbar_wait(&empty_bar[g % C::kStages], ((g / C::kStages) & 1) ^ 1,
                                                   deadline, &abort_sh)) {
          record_error(args.err, kErrTimeout);
          abort_sh = 1;
        }
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      // ---------------------------------------------- MMA (even CTA) ----
      constexpr uint32_t idesc_dn = idesc_nvf4(256, C::BN, false);
      constexpr uint32_t idesc_sp = idesc_nvf4(256, C::BN, true);
      uint32_t g = 0, k = 0;
      for (int tile = pair; tile < ntiles && !abort_sh; tile += npairs) {
        const uint64_t deadline = globaltimer_ns() + kWaitLimitNs;
        if (k > 0 && !mbar_wait_cluster(&acc_empty, (k - 1) & 1, deadline, &abort_sh)) {
          record_error(args.err, kErrTimeout);
          abort_sh = 1;
          break;
        }
        tc_fence_after();
        for (int i = 0; i < KS; ++i, ++g) {
          const int s = g % C::kStages, r = g % C::kRegions;
          const uint32_t ph = (g / C::kStages) & 1;
          if (!mbar_wait(&full_bar[s], ph, deadline, &abort_sh) ||
              !mbar_wait_cluster(&peer_full[s], ph, deadline, &abort_sh) ||
              !mbar_wait(&sf_full[r], (g / C::kRegions) & 1, deadline, &abort_sh)) {
            record_error(args.err, kErrTimeout);
            abort_sh = 1;
            break;
          }
          tc_fence_after();
          const uint32_t st = smem_u32(smem + s * C::kStageBytes);
          const uint32_t sf = tmem + C::kColSf0 + (uint32_t)r * C::kSfRegion;
          if (C::kHas1) {
#pragma unroll
            for (int j = 0; j < 2; ++j)
              mma_pair_sp_nvf4(tmem + C::kColAcc, smem_desc(st + C::kOffA1 + 32 * j, 16, 512, kSw64),
                               smem_desc(st + C::kOffB + 64 * j, 16, 1024, kSw128), sf + C::kSfE1 + 2 * j, idesc_sp,
                               sf + C::kSfS1 + 4 * j, sf + C::kSfB32 + j * C::kSfbCols, (i > 0 || j > 0) ? 1u : 0u);
          }
#pragma unroll
          for (int j = 0; j < 4; ++j)
            mma_pair_nvf4(tmem + C::kColAcc, smem_desc(st + C::kOffA2 + 32 * j, 16, 1024, kSw128),
                          smem_desc(st + C::kOffB + 32 * j, 16, 1024, kSw128), idesc_dn, sf + C::kSfS2 + 4 * j,
                          sf + C::kSfB16 + j * C::kSfbCols, (C::kHas1 || i > 0 || j > 0) ? 1u : 0u);
          tc_commit_pair_mc(&empty_bar[s], 0x3);  // both CTAs' ring slot s
          tc_commit_pair(&region_free[r]);        // the scale region, for the copy warps
        }
        tc_commit_pair_mc(&acc_full, 0x3);        // both CTAs' accumulator rows
        ++k;
      }
    } else if (lane == 0) {
      // ------------------------- odd CTA: forward "stage landed" ----
      uint32_t g = 0;
      for (int tile = pair; tile < ntiles && !abort_sh; tile += npairs) {
        const uint64_t deadline = globaltimer_ns() + kWaitLimitNs;
        for (int i = 0; i < KS; ++i, ++g) {
          const int s = g % C::kStages;
          if (!mbar_wait(&full_bar[s], (g / C::kStages) & 1, deadline, &abort_sh)) {
            record_error(args.err, kErrTimeout);
            abort_sh = 1;
            break;
          }
          // the stage's bytes are in this CTA's shared memory (its barrier
          // completed); the even CTA's copies and MMAs read them after its
          // wait on peer_full, so the arrival need not order anything
          mbar_arrive_remote_relaxed(peer_full_lead + (uint32_t)(s * sizeof(uint64_t)));
        }
      }
    }
  } else if (cw >= 0) {
    if (lane == 0 && leader) {
      // ----------------------------------------- copy warps (even CTA) ----
      uint32_t g = 0;
      for (int tile = pair; tile < ntiles && !abort_sh; tile += npairs) {
        const uint64_t deadline = globaltimer_ns() + kWaitLimitNs;
        for (int i = 0; i < KS; ++i, ++g) {
          const int s = g % C::kStages, r = g % C::kRegions;
          const uint32_t ph = (g / C::kStages) & 1;
          // both CTAs' stage data has landed, and the MMAs of stage g - 3
          // (the region's previous user) have completed
          if (!mbar_wait(&full_bar[s], ph, deadline, &abort_sh) ||
              !mbar_wait_cluster(&peer_full[s], ph, deadline, &abort_sh) ||
              (g >= (uint32_t)C::kRegions &&
               !mbar_wait(&region_free[r], ((g / C::kRegions) & 1) ^ 1, deadline, &abort_sh))) {
            record_error(args.err, kErrTimeout);
            abort_sh = 1;
            break;
          }
          tc_fence_after();
          const uint32_t st = smem_u32(smem + s * C::kStageBytes);
          const uint32_t sf = tmem + C::kColSf0 + (uint32_t)r * C::kSfRegion;
          int n = 0;
          auto cp4 = [&](uint32_t taddr, uint32_t saddr) {
            if (n++ % C::kCW == cw) tc_cp_pair_32x128b_x4(taddr, smem_desc(saddr, 0, 128, kSwNone));
          };
#pragma unroll
          for (int j = 0; j < 4; ++j)
#pragma unroll
            for (int h = 0; h < 2; ++h) cp4(sf + C::kSfB16 + j * C::kSfbCols + 4 * h, st + C::kOffSFB16 + h * kSf16Tile + 512 * j);
          if (C::kHas1) {
#pragma unroll
            for (int j = 0; j < 2; ++j)
#pragma unroll
              for (int h = 0; h < 2; ++h)
                cp4(sf + C::kSfB32 + j * C::kSfbCols + 4 * h, st + C::kOffSFB32 + h * kSf32Tile + 512 * j);
            if (n++ % C::kCW == cw) tc_cp_pair_128x128b(sf + C::kSfE1, smem_desc(st + C::kOffE1, 0, 128, kSwNone));
#pragma unroll
            for (int j = 0; j < 2; ++j) cp4(sf + C::kSfS1 + 4 * j, st + C::kOffS1 + 512 * j);
          }
#pragma unroll
          for (int j = 0; j < 4; ++j) cp4(sf + C::kSfS2 + 4 * j, st + C::kOffS2 + 512 * j);
          tc_commit_pair(&sf_full[r]);
        }
      }
      tc_commit_pair(&cp_fin[cw]);
      const uint64_t lim = globaltimer_ns() + kWaitLimitNs;
      while (!mbar_try_wait(&cp_fin[cw], 0) && globaltimer_ns() < lim) {
      }
    }
  }
  } else {
    // ---------------------------------------------- epilogue (both) ----
    regs_inc_epi();  // the epilogue warpgroup holds a 256-column row
    const int sp = warp & 3;  // TMEM lane quarter this warp may access
    const int rl = sp * 32 + lane;
    grid_dependency_wait();  // s_g is written by the preceding sharq_prep
    const float s_tensor = args.per_token ? 0.0f : *args.s_g;
    const float s_w = args.s_w[0];
    uint32_t k = 0;
    for (int tile = pair; tile < ntiles && !abort_sh; tile += npairs) {
      int m2, nt;
      tile_coords(tile, m2_tiles, n_tiles, args.n_major, m2, nt);
      const int mt = 2 * m2 + (int)rank;
      const int valid = max(0, min(128, args.T - mt * 128));
      const uint64_t deadline = globaltimer_ns() + kWaitLimitNs;
      if (!mbar_wait_cluster(&acc_full, k & 1, deadline, &abort_sh)) {
        record_error(args.err, kErrTimeout);
        abort_sh = 1;
        break;
      }
      tc_fence_after();
      const int row = mt * 128 + rl;
      const float scale = __fmul_rn(args.per_token ? (rl < valid ? args.s_g[row] : 0.0f) : s_tensor, s_w);
      const size_t off = (size_t)row * args.D + (size_t)nt * C::BN;
      if (!args.out_f32) {
        uint32_t pk[C::BN / 2];  // the row as packed bf16, then the accumulator is free
#pragma unroll
        for (int c = 0; c < C::BN; c += 64) {  // two loads in flight per wait
          uint32_t v[2][32];
          tmem_ld32(tmem + ((uint32_t)(sp * 32) << 16) + C::kColAcc + c, v[0]);
          tmem_ld32(tmem + ((uint32_t)(sp * 32) << 16) + C::kColAcc + c + 32, v[1]);
          tmem_ld_wait();
#pragma unroll
          for (int q = 0; q < 32; ++q) {
            __nv_bfloat162 b2 = __floats2bfloat162_rn(__fmul_rn(__uint_as_float(v[q >> 4][2 * (q & 15)]), scale),
                                                      __fmul_rn(__uint_as_float(v[q >> 4][2 * (q & 15) + 1]), scale));
            pk[c / 2 + q] = *reinterpret_cast<uint32_t*>(&b2);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_remote_relaxed(acc_empty_lead);  // loads done: one arrival per warp, 8 per tile
        store_rows_bf16_staged<C::BN>(pk, smem + C::kOffStage + (size_t)sp * 4096,
                                      static_cast<__nv_bfloat16*>(args.Y) + (size_t)(mt * 128 + sp * 32) * args.D +
                                          (size_t)nt * C::BN,
                                      (size_t)args.D, valid - sp * 32, lane);
      } else {
#pragma unroll 1
        for (int c = 0; c < C::BN; c += 32) {
          uint32_t v[32];
          tmem_ld32(tmem + ((uint32_t)(sp * 32) << 16) + C::kColAcc + c, v);
          tmem_ld_wait();
          if (rl < valid) store_row32(args.Y, 1, off + c, v, scale);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_remote_relaxed(acc_empty_lead);
      }
      ++k;
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // neither CTA frees its TMEM or leaves while the pair's work may touch it
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, C::kTmemCols);
  }
}

// The pair kernel's register split (setmaxnreg) needs the launch to hold the
// full 65536 registers / 512 threads; a build whose kernel was allotted fewer
// would make the epilogue's increase wait for registers that never come, so
// the launcher checks and otherwise uses the one-CTA kernel.
template <int kG>
bool pair_regs_ok() {
  cudaFuncAttributes fa{};
  if (cudaFuncGetAttributes(&fa, sharq_gemm_pair_kernel<kG>) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  using C = PairCfg<kG>;
  return fa.numRegs * C::kThreadsT >= 128 * (C::kRegsEpi + 3 * C::kRegsOther);
}

template <int kG>
cudaError_t launch_pair(const GemmArgs& a, int m_tiles, cudaStream_t stream, bool* launched) {
  using C = PairCfg<kG>;
  static int sms[64] = {};  // SM count, or -1 if this device cannot run the pair form
  *launched = false;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 64) return cudaErrorInvalidDevice;
  if (sms[dev] == 0) {
    if (!pair_regs_ok<kG>()) {
      sms[dev] = -1;
    } else {
      e = cudaFuncSetAttribute(sharq_gemm_pair_kernel<kG>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               C::kSmemBytes);
      if (e != cudaSuccess) return e;
      int n = 0;
      e = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
      if (e != cudaSuccess) return e;
      sms[dev] = n;
    }
  }
  if (sms[dev] < 2) return cudaSuccess;
  const long long ntiles = (long long)((m_tiles + 1) / 2) * (a.D / C::BN);
  const long long pairs = ntiles < sms[dev] / 2 ? ntiles : sms[dev] / 2;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(2 * pairs));
  cfg.blockDim = dim3(C::kThreadsT);
  cfg.dynamicSmemBytes = C::kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = 2;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  e = cudaLaunchKernelEx(&cfg, sharq_gemm_pair_kernel<kG>, a, m_tiles);
  *launched = e == cudaSuccess;
  return e;
}

template <int BN, int kG>
cudaError_t launch_persistent(const GemmArgs& a, int m_tiles, cudaStream_t stream) {
  using C = PCfg<BN, kG>;
  static int sms[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 64) return cudaErrorInvalidDevice;
  if (sms[dev] == 0) {
    e = cudaFuncSetAttribute(sharq_gemm_persistent_kernel<BN, kG>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             C::kSmemBytes);
    if (e != cudaSuccess) return e;
    int n = 0;
    e = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    sms[dev] = n;
  }
  const long long ntiles = (long long)m_tiles * (a.D / BN);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(ntiles < sms[dev] ? ntiles : sms[dev]));
  cfg.blockDim = dim3(C::kThreadsT);
  cfg.dynamicSmemBytes = C::kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, sharq_gemm_persistent_kernel<BN, kG>, a, m_tiles);
}

template <int BN>
cudaError_t launch_persistent_mode(const GemmArgs& a, int m_tiles, int gmode, cudaStream_t stream) {
  switch (gmode) {
    case kGemmSharq: return launch_persistent<BN, kGemmSharq>(a, m_tiles, stream);
    case kGemmNvfp4: return launch_persistent<BN, kGemmNvfp4>(a, m_tiles, stream);
    case kGemmSparseOnly: return launch_persistent<BN, kGemmSparseOnly>(a, m_tiles, stream);
    case kGemmDenseDense: return launch_persistent<BN, kGemmDenseDense>(a, m_tiles, stream);
    case kGemmSparseSparse: return launch_persistent<BN, kGemmSparseSparse>(a, m_tiles, stream);
    case kGemmSharqMx: return launch_persistent<BN, kGemmSharqMx>(a, m_tiles, stream);
    case kGemmMxfp4: return launch_persistent<BN, kGemmMxfp4>(a, m_tiles, stream);
    default: return cudaErrorInvalidValue;
  }
}

template <int BN, bool kSplit, bool kFused>
cudaError_t launch_cfg(const GemmArgs& a, int m_tiles, cudaStream_t stream) {
  using C = Cfg<BN, kSplit, kFused>;
  static bool attr_set[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 64 && !attr_set[dev]) {
    e = cudaFuncSetAttribute(sharq_gemm_kernel<BN, kSplit, kFused>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             C::kSmemBytes);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(a.D / BN, m_tiles, kSplit ? a.splits : 1);
  cfg.blockDim = dim3(C::kThreadsT);
  cfg.dynamicSmemBytes = C::kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = 1;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = kSplit ? a.splits : 1;
  cfg.attrs = attr;
  cfg.numAttrs = kSplit ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, sharq_gemm_kernel<BN, kSplit, kFused>, a);
}

}  // namespace

// Clusters of the split-K decode kernel (1 x 1 x splits CTAs) that can be
// resident at once on this device: clusters must fit within one GPC, so
// clusters of 4 leave SMs of each GPC idle, and a grid with more clusters
// than this runs in two waves.  Cached per device, form and split count;
// 0 if the query fails.
int split_max_clusters(int splits, bool fused) {
  static int cache[64][2][5] = {};
  int dev = 0;
  if (splits < 2 || splits > 4 || cudaGetDevice(&dev) != cudaSuccess || dev >= 64) return 0;
  int& c = cache[dev][fused ? 1 : 0][splits];
  if (c == 0) {
    auto fn = fused ? sharq_gemm_kernel<128, true, true> : sharq_gemm_kernel<128, true, false>;
    const int smem = fused ? Cfg<128, true, true>::kSmemBytes : Cfg<128, true, false>::kSmemBytes;
    const int threads = fused ? Cfg<128, true, true>::kThreadsT : Cfg<128, true, false>::kThreadsT;
    int n = 0;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(1, 1, splits);
    cfg.blockDim = dim3(threads);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 1;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = splits;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess ||
        cudaOccupancyMaxActiveClusters(&n, fn, &cfg) != cudaSuccess || n < 1) {
      cudaGetLastError();
      n = -1;
    }
    c = n;
  }
  return c > 0 ? c : 0;
}

// The CTA-pair prefill form is on unless the environment sets
// SHARQ_GEMM_PAIR=0 (read once per process), which runs those shapes on the
// one-CTA persistent kernel instead -- the same result, for comparing the two.
bool pair_form_enabled() {
  static const bool on = [] {
    const char* v = getenv("SHARQ_GEMM_PAIR");
    return !(v && v[0] == '0');
  }();
  return on;
}

#ifdef SHARQ_TRACE
extern "C" int sharq_debug_set_trace(void* p) {
  return cudaMemcpyToSymbol(g_trace, &p, sizeof(p)) == cudaSuccess ? 0 : -4;
}
#endif

cudaError_t launch_linear(const uint8_t* a_sp, const uint8_t* a_meta, const uint8_t* a_spsf, const uint8_t* a_r,
                          const uint8_t* a_rsf, const uint8_t* a_rmeta, const float* s_g, int T, int Tp, int K,
                          int gmode,
                          const uint8_t* w_codes, const uint8_t* w_sf32, const uint8_t* w_sf16, const float* s_w,
                          int D, int E, const int* group_offsets, void* Y, int out_f32, int bn, int splits,
                          int* err, const int* act_err, cudaStream_t stream, const void* X_fused,
                          const void* gamma_fused, float eps_fused, bool per_token) {
  GemmArgs a = {};
  a.a_sp = a_sp;
  a.a_meta = a_meta;
  a.a_spsf = a_spsf;
  a.a_r = a_r;
  a.a_rsf = a_rsf;
  a.a_rmeta = a_rmeta;
  a.s_g = s_g;
  a.w_codes = w_codes;
  a.w_sf32 = w_sf32;
  a.w_sf16 = w_sf16;
  a.s_w = s_w;
  a.Y = Y;
  a.group_offsets = group_offsets;
  a.err = err;
  a.act_err = act_err;
  a.T = T;
  a.K = K;
  a.D = D;
  a.E = E;
  a.out_f32 = out_f32;
  a.sharq_mode = gmode == kGemmSharq ? 1 : 0;
  const bool two_way = gmode == kGemmSharq || gmode == kGemmNvfp4;  // the split-K/fused kernels' modes
  a.splits = splits;
  a.per_token = per_token ? 1 : 0;
  a.X = static_cast<const __nv_bfloat16*>(X_fused);
  a.gamma = static_cast<const __nv_bfloat16*>(gamma_fused);
  a.eps = eps_fused;
  const int m_tiles = Tp / 128;
  if (m_tiles == 0) return cudaSuccess;
  // keep the smaller operand resident in L2: column-tile major order when the
  // packed weight (0.59375 B per element) outweighs the prepared activation
  // (0.90625 B per element of the padded rows).  Grouped experts keep row
  // order: consecutive row tiles of one expert share its (small) weight.
  a.n_major = (!group_offsets && (double)D * 0.59375 > (double)Tp * 0.90625) ? 1 : 0;
  if (X_fused) {  // fused decode form
    if (T > 32 || m_tiles != 1 || gmode != kGemmSharq || group_offsets || per_token) return cudaErrorInvalidValue;
    if (splits > 1) {
      if (bn != 128 || splits > 4) return cudaErrorInvalidValue;
      return launch_cfg<128, true, true>(a, m_tiles, stream);
    }
    return bn == 256 ? launch_cfg<256, false, true>(a, m_tiles, stream)
                     : launch_cfg<128, false, true>(a, m_tiles, stream);
  }
  if (splits > 1 && two_way) {
    if (bn != 128 || splits > 4) return cudaErrorInvalidValue;
    return launch_cfg<128, true, false>(a, m_tiles, stream);
  }
  // prefill SharQ / plain-NVFP4 GEMMs with two or more 128-row tiles and
  // 256-column tiles: the CTA-pair form
  if (two_way && !group_offsets && E == 1 && m_tiles >= 2 && bn == 256 && a.D % 256 == 0 && pair_form_enabled()) {
    bool launched = false;
    const cudaError_t e = gmode == kGemmSharq ? launch_pair<kGemmSharq>(a, m_tiles, stream, &launched)
                                              : launch_pair<kGemmNvfp4>(a, m_tiles, stream, &launched);
    if (e != cudaSuccess || launched) return e;
  }
  // the Table-5 modes run the persistent form at every size
  const int pbn = (a.D % 256 == 0) ? 256 : 128;
  const int use_bn = two_way ? bn : pbn;
  return use_bn == 256 ? launch_persistent_mode<256>(a, m_tiles, gmode, stream)
                       : launch_persistent_mode<128>(a, m_tiles, gmode, stream);
}

}  // namespace sharq
