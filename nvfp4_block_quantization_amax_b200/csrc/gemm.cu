// gemm.cu -- block-scaled NVFP4 (and MXFP4) GEMM on the sm_100a tensor cores.
//
//   D[m, n] = alphaA * alphaB * sum_k (qA[m,k] DeltaA[m,k/16]) (qB[n,k] DeltaB[n,k/16])
//
// MXFP4 operands (UE8M0 scales per 32 K, no tensor scales) run through the
// CTA-pair kernel with MX = true: the same pipeline, .block32 MMAs, one scale
// atom per two MMAs.
//
// The NVFP4 pretraining write-up (§四) describes the Blackwell tensor cores
// that read narrow values plus 8-bit block scales and accumulate in FP32; this
// kernel drives them directly:
//   * warp 0 (one lane, elected once, running the whole loop): TMA producer.  Per K-stage of 256 elements it loads
//     the A tile (128 rows x 128 B) and the B tile (BN rows x 128 B) with 128-
//     byte swizzle, and the matching scale atoms (512 B per 128 rows x 64 K)
//     with bulk copies, into a ring of shared-memory stages guarded by
//     mbarriers.
//   * warp 1: allocates tensor memory; one elected lane copies each stage's scales
//     into TMEM (tcgen05.cp 32x128b.warpx4) and issues four
//     tcgen05.mma.kind::mxf4nvf4.block_scale.block16 (M=128, N=BN, K=64),
//     accumulating in TMEM, then commits the stage back to the producer.
//   * warps 2-5: epilogue.  Each reads its 32-lane quarter of the FP32
//     accumulator with tcgen05.ld, multiplies by alphaA * alphaB and converts
//     to bf16 into registers (the whole row), hands the accumulator back, then
//     writes 16-row x 128-byte boxes into swizzled shared memory and stores
//     them with TMA.
// The kernel is persistent (one CTA per SM, tiles round-robin): the producer
// runs ahead into the next tile while the epilogue drains the accumulator,
// and the MMA warp starts the next tile as soon as the accumulator is read.
// Every wait is bounded (about two seconds of %globaltimer); a wait that
// gives up raises an abort flag that every role checks, the kernel records
// NVFP4_ERR_TIMEOUT in the optional status word and still frees its TMEM.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "nvfp4_device.cuh"
#include "launch.cuh"
#include "nvfp4_internal.h"

namespace nvfp4 {
namespace {

constexpr int BM = 128;
constexpr int BK_BYTES = 128;  // 256 FP4 values per row per stage: four MMA K blocks
constexpr int KB_PER_STAGE = 4;
constexpr int kOutStaging = 4 * 2048;  // epilogue: one 16-row x 128-byte box per warp
constexpr int kSfSlots = 2 * KB_PER_STAGE;  // TMEM scale slots: two sets of one stage's K blocks
constexpr int NUM_THREADS = 192;
constexpr uint64_t kTimeoutNs = 2000000000ull;

template <int BN>
struct Cfg {
  static constexpr int A_STAGE = BM * BK_BYTES;
  static constexpr int B_STAGE = BN * BK_BYTES;
  static constexpr int SFA_STAGE = KB_PER_STAGE * 512;
  static constexpr int SFB_STAGE = (BN / 128) * KB_PER_STAGE * 512;
  static constexpr int STAGE = A_STAGE + B_STAGE + SFA_STAGE + SFB_STAGE;
  // as many stages as fit: loads take about a microsecond to land, so the
  // ring must hold that much MMA work
  static constexpr int STAGES = (232448 - kOutStaging - 1024 - 512) / STAGE;
  static constexpr int SMEM = STAGES * STAGE + kOutStaging + 1024 /* alignment */ + 512 /* barriers */;
  // Scales of one 64-wide K block in TMEM: SFA 4 columns, then SFB
  // 4 * (BN / 128) columns.
  static constexpr uint32_t SF_W = 4 + 4 * (BN / 128);
  static constexpr uint32_t TMEM_COLS = (BN + kSfSlots * SF_W) <= 256 ? 256 : 512;
  static constexpr uint32_t SF_COL = BN;
  // Instruction descriptor (kind::mxf4nvf4): A and B are E2M1 (format 1),
  // K-major, scales E4M3, N >> 3 at bit 17, M >> 4 at bit 24.
  static constexpr uint32_t IDESC = (1u << 7) | (1u << 10) | ((uint32_t(BN) >> 3) << 17) | ((uint32_t(BM) >> 4) << 24);
};

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// One lane of a converged warp (elect.sync): the warp computes every operand
// together so they stay warp-uniform, and this lane issues the single-thread
// tcgen05 / TMA instruction.
__device__ __forceinline__ bool elect_one() {
  uint32_t pred = 0;
  asm volatile(
      "{\n\t.reg .b32 r;\n\t.reg .pred p;\n\t"
      "elect.sync r|p, 0xffffffff;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(pred));
  return pred != 0;
}

__device__ __forceinline__ uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Wait for the phase with the given parity; false if the abort flag is up or
// the wait ran past the time limit (which raises the flag).
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (globaltimer() - t0 > kTimeoutNs) {
      *abort_flag = 1;
      return false;
    }
  }
}

// Bounded wait for the first phase of `bar` (used only after an abort, where
// the abort flag is already up).
__device__ __forceinline__ void mbar_wait_bounded(uint32_t bar, uint32_t parity) {
  const uint64_t t0 = globaltimer();
  while (!mbar_try_wait(bar, parity) && globaltimer() - t0 < kTimeoutNs) {
  }
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
      : "memory");
}

__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(src), "r"(bytes), "r"(bar)
               : "memory");
}

// Shared-memory matrix descriptor, K-major operand with 128-byte swizzle:
// start >> 4, leading offset 1 (unused when swizzled), stride 1024 B between
// 8-row groups (8 rows x 128 B), descriptor version 1, layout SWIZZLE_128B
// (2) in bits 61-63.
__device__ __forceinline__ uint64_t desc_sw128(uint32_t addr) {
  return static_cast<uint64_t>((addr >> 4) & 0x3FFFu) | (1ull << 16) | (static_cast<uint64_t>(1024 >> 4) << 32) |
         (1ull << 46) | (2ull << 61);
}

// Descriptor of a 32 x 16-byte scale atom (no swizzle, 8-row groups 128 B
// apart) for tcgen05.cp.
__device__ __forceinline__ uint64_t desc_sf(uint32_t addr) {
  return static_cast<uint64_t>((addr >> 4) & 0x3FFFu) | (static_cast<uint64_t>(128 >> 4) << 32) | (1ull << 46);
}

__device__ __forceinline__ void mma_mxf4nvf4(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                             uint32_t accumulate, uint32_t tsfa, uint32_t tsfb) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(tsfa), "r"(tsfb)
      : "memory");
}

__device__ __forceinline__ void tmem_cp_sf(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

__device__ __forceinline__ void umma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// 32 lanes x 32 columns of 32-bit accumulators: thread t gets lane t's row
// (the caller waits with tmem_ld_wait before using r).
__device__ __forceinline__ void tmem_ld32_nowait(uint32_t taddr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]),
        "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}

__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Relaxed CTA-local arrive (the accumulator hand-back; see mbar_arrive_cluster).
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.relaxed.cta.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// TMA tile store from shared memory (bulk-group completion).
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, uint32_t src, int x, int y) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(src), "r"(x), "r"(y)
               : "memory");
}

__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }

template <int N>
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }


// ---- cluster / CTA-pair helpers (2-SM MMA) ----
__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release;\n\tbarrier.cluster.wait.acquire;" ::: "memory");
}

// shared::cluster address of the same shared-memory location in CTA `rank`
__device__ __forceinline__ uint32_t map_to_rank(uint32_t local_addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(local_addr), "r"(rank));
  return r;
}

// Epilogue hand-back of the accumulator to the leader CTA's barrier.  The
// arrive is relaxed: the accumulator reads it guards have completed into
// registers (tcgen05.wait::ld) and are ordered before it by
// tcgen05.fence::before_thread_sync, and nothing in memory is published
// through it.  A release at cluster scope here cost about 1100 cycles per
// tile on B200 (it waits for the thread's outstanding memory operations).
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.relaxed.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}

// TMA tile load into this CTA's shared memory whose completion is counted on
// an mbarrier that may live in the peer CTA of the pair (no multicast).
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap* map, int x, int y,
                                                 uint32_t bar_cluster) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], "
      "[%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar_cluster)
      : "memory");
}

__device__ __forceinline__ void mma_mxf4nvf4_pair(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                                  uint32_t accumulate, uint32_t tsfa, uint32_t tsfb) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(tsfa), "r"(tsfb)
      : "memory");
}

// MXFP4 operands: E2M1 values with UE8M0 scales per 32 K (two scale bytes per
// row per K = 64 MMA, chosen inside each 32-bit TMEM scale column by the
// descriptor's scale-factor ids).
__device__ __forceinline__ void mma_mxf4_pair(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                              uint32_t accumulate, uint32_t tsfa, uint32_t tsfb) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.block32 [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(tsfa), "r"(tsfb)
      : "memory");
}

__device__ __forceinline__ void tmem_cp_sf_pair(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::2.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

// Arrive on the mbarrier at this shared-memory offset in both CTAs of the pair
// once every tcgen05 operation issued so far has completed.
__device__ __forceinline__ void umma_commit_pair(uint32_t bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(bar),
      "h"(static_cast<uint16_t>(0x3))
      : "memory");
}

template <int BN>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    nvfp4_gemm_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
                      const __grid_constant__ CUtensorMap tmap_d, const uint8_t* __restrict__ sfa,
                      const uint8_t* __restrict__ sfb, const float* __restrict__ alpha_a,
                      const float* __restrict__ alpha_b, int M, int N, int K, int out_fp32, int32_t* status) {
  pdl_entry();
  using G = Cfg<BN>;
  constexpr int STAGES = G::STAGES;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = sA + STAGES * G::A_STAGE;
  uint8_t* sSFA = sB + STAGES * G::B_STAGE;
  uint8_t* sSFB = sSFA + STAGES * G::SFA_STAGE;
  uint8_t* sOut = sSFB + STAGES * G::SFB_STAGE;  // 4 warps x one 2 KB box, 1024-aligned
  uint64_t* bars = reinterpret_cast<uint64_t*>(sOut + kOutStaging);
  uint64_t* full = bars;
  uint64_t* empty = bars + STAGES;
  uint64_t* acc_full = bars + 2 * STAGES;
  uint64_t* acc_empty = bars + 2 * STAGES + 1;
  uint64_t* drain = bars + 2 * STAGES + 2;   // tensor-op drain after an abort
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * STAGES + 3);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m_tiles = M / BM;
  const int num_tiles = m_tiles * (N / BN);
  const int kblocks64 = K / 64;  // scale atoms along K
  const int kstages = (K + 255) / 256;  // K % 128 == 0: the last stage may hold 2 K blocks

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), 1);
    }
    mbar_init(smem_u32(acc_full), 1);
    mbar_init(smem_u32(acc_empty), 4);  // one arrival per epilogue warp
    mbar_init(smem_u32(drain), 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(G::TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  fence_before();
  __syncthreads();
  fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ---------------- producer: runs ahead across tiles ----------------
    // One lane, elected once, walks every stage and issues the copies.
    if (elect_one()) {
      int it = 0;  // global stage counter
      bool stop = false;
      for (int tile = blockIdx.x; tile < num_tiles && !stop; tile += gridDim.x) {
        const int tile_m = tile % m_tiles, tile_n = tile / m_tiles;
        for (int kt = 0; kt < kstages; ++kt, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1;
          if (!mbar_wait(smem_u32(&empty[s]), ph ^ 1, abort_flag)) {
            stop = true;
            break;
          }
          const int nk = min(KB_PER_STAGE, kblocks64 - KB_PER_STAGE * kt);  // K blocks in this stage
          const uint32_t bytes = G::A_STAGE + G::B_STAGE + nk * 512 * (1 + BN / 128);
          const uint32_t fb = smem_u32(&full[s]);
          const uint32_t dA = smem_u32(sA + s * G::A_STAGE), dB = smem_u32(sB + s * G::B_STAGE);
          const uint32_t dSA = smem_u32(sSFA + s * G::SFA_STAGE), dSB = smem_u32(sSFB + s * G::SFB_STAGE);
          const uint8_t* gSA = sfa + (static_cast<int64_t>(tile_m) * kblocks64 + KB_PER_STAGE * kt) * 512;
          mbar_expect_tx(fb, bytes);
          tma_load_2d(dA, &tmap_a, kt * BK_BYTES, tile_m * BM, fb);
          tma_load_2d(dB, &tmap_b, kt * BK_BYTES, tile_n * BN, fb);
          bulk_load(dSA, gSA, nk * 512, fb);
#pragma unroll
          for (int g = 0; g < BN / 128; ++g)
            bulk_load(dSB + g * KB_PER_STAGE * 512,
                      sfb + (static_cast<int64_t>(tile_n * (BN / 128) + g) * kblocks64 + KB_PER_STAGE * kt) * 512,
                      nk * 512, fb);
        }
      }
      if (*abort_flag) {
        // A wait gave up somewhere: let the copies already issued land before
        // the CTA exits (each wait again bounded).
        for (int i = (it > STAGES ? it - STAGES : 0); i < it; ++i) {
          const uint32_t bar = smem_u32(&full[i % STAGES]), ph = (i / STAGES) & 1;
          mbar_wait_bounded(bar, ph);
        }
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer (one lane, elected once) ----------------
    // Per stage: wait for its data, copy its scales (one TMEM slot per K
    // block, two slot sets used alternately so the copies never overwrite
    // scales an earlier, still-running MMA reads), issue its MMAs, release
    // the stage.
    if (elect_one()) {
      const int my_tiles = (num_tiles - static_cast<int>(blockIdx.x) + static_cast<int>(gridDim.x) - 1) /
                           static_cast<int>(gridDim.x);
      const int total = my_tiles * kstages;
      for (int g = 0; g < total; ++g) {
        const int kt = g % kstages, ti = g / kstages, s = g % STAGES;
        if (kt == 0) {
          // the epilogue must have drained the previous tile's accumulator
          if (!mbar_wait(smem_u32(acc_empty), (ti & 1) ^ 1, abort_flag)) break;
          fence_after();
        }
        if (!mbar_wait(smem_u32(&full[s]), (g / STAGES) & 1, abort_flag)) break;
        fence_after();
        const uint32_t sfa_s = smem_u32(sSFA + s * G::SFA_STAGE);
        const uint32_t sfb_s = smem_u32(sSFB + s * G::SFB_STAGE);
        const uint32_t set = static_cast<uint32_t>(g & 1) * KB_PER_STAGE;
        const int nk = min(KB_PER_STAGE, kblocks64 - KB_PER_STAGE * kt);
        const uint64_t adesc = desc_sw128(smem_u32(sA + s * G::A_STAGE));
        const uint64_t bdesc = desc_sw128(smem_u32(sB + s * G::B_STAGE));
        // each K block's scales are copied right before its MMA (interleaved)
        for (int kk = 0; kk < nk; ++kk) {
          const uint32_t col = tmem + G::SF_COL + (set + kk) * G::SF_W;
          tmem_cp_sf(col, desc_sf(sfa_s + 512 * kk));
#pragma unroll
          for (int gg = 0; gg < BN / 128; ++gg)
            tmem_cp_sf(col + 4 + 4 * gg, desc_sf(sfb_s + gg * KB_PER_STAGE * 512 + 512 * kk));
          // K = 64 FP4 values = 32 bytes: advance the start address by 2 x 16 B
          mma_mxf4nvf4(tmem, adesc + 2 * kk, bdesc + 2 * kk, G::IDESC, (kt > 0 || kk > 0) ? 1u : 0u, col, col + 4);
        }
        umma_commit(smem_u32(&empty[s]));
        if (kt == kstages - 1) umma_commit(smem_u32(acc_full));
      }
      if (*abort_flag) {
        // a wait gave up: the copies and MMAs already issued may still run;
        // let them finish (bounded) before TMEM is freed
        umma_commit(smem_u32(drain));
        mbar_wait_bounded(smem_u32(drain), 0);
      }
    }
  } else {
    // ---------------- epilogue (warps 2..5) ----------------
    // Warp w reads TMEM lanes 32 (w % 4) .. + 31 = output rows of the tile.
    // bf16: the whole 256-column row goes to registers as packed bf16 first,
    // so the accumulator is handed back to the MMA warp before any store;
    // then 16-row x 128-byte boxes go out through one swizzled staging
    // buffer per warp with TMA stores.
    const int q = warp & 3;
    uint8_t* buf = sOut + (warp - 2) * 2048;
    const float ab = __fmul_rn(__ldg(alpha_a), __ldg(alpha_b));
    int ti = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++ti) {
      const int tile_m = tile % m_tiles, tile_n = tile / m_tiles;
      if (!mbar_wait(smem_u32(acc_full), ti & 1, abort_flag)) break;
      fence_after();
      const int row0 = tile_m * BM + 32 * q;
      const uint32_t taddr = tmem + (static_cast<uint32_t>(32 * q) << 16);
      if (!out_fp32) {
        uint32_t packed[BN / 2];
#pragma unroll
        for (int c = 0; c < BN; c += 32) {
          uint32_t r[32];
          tmem_ld32_nowait(taddr + c, r);
          tmem_ld_wait();
#pragma unroll
          for (int h = 0; h < 16; ++h) {
            const __nv_bfloat162 b2 = __floats2bfloat162_rn(__fmul_rn(__uint_as_float(r[2 * h]), ab),
                                                            __fmul_rn(__uint_as_float(r[2 * h + 1]), ab));
            packed[c / 2 + h] = *reinterpret_cast<const uint32_t*>(&b2);
          }
        }
        fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(acc_empty));
#pragma unroll
        for (int p = 0; p < BN / 64; ++p) {      // 64-column pieces
#pragma unroll
          for (int half = 0; half < 2; ++half) {  // rows 0-15, 16-31 of the warp
            if (lane == 0) bulk_wait_read<0>();  // the previous box has been read
            __syncwarp();
            if ((lane >> 4) == half) {
              uint8_t* rowp = buf + (lane & 15) * 128;
#pragma unroll
              for (int j = 0; j < 8; ++j)
                *reinterpret_cast<uint4*>(rowp + ((j ^ (lane & 7)) << 4)) =
                    make_uint4(packed[32 * p + 4 * j], packed[32 * p + 4 * j + 1], packed[32 * p + 4 * j + 2],
                               packed[32 * p + 4 * j + 3]);
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              tma_store_2d(&tmap_d, smem_u32(buf), tile_n * BN + 64 * p, row0 + 16 * half);
              bulk_commit();
            }
          }
        }
      } else {
        // fp32: 32-column pieces straight from TMEM
#pragma unroll 1
        for (int c = 0; c < BN; c += 32) {
          uint32_t r[32];
          tmem_ld32_nowait(taddr + c, r);
          tmem_ld_wait();
          if (c + 32 == BN) {
            fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(acc_empty));
          }
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            if (lane == 0) bulk_wait_read<0>();
            __syncwarp();
            if ((lane >> 4) == half) {
              uint8_t* rowp = buf + (lane & 15) * 128;
#pragma unroll
              for (int j = 0; j < 8; ++j)
                *reinterpret_cast<uint4*>(rowp + ((j ^ (lane & 7)) << 4)) =
                    make_uint4(__float_as_uint(__fmul_rn(__uint_as_float(r[4 * j]), ab)),
                               __float_as_uint(__fmul_rn(__uint_as_float(r[4 * j + 1]), ab)),
                               __float_as_uint(__fmul_rn(__uint_as_float(r[4 * j + 2]), ab)),
                               __float_as_uint(__fmul_rn(__uint_as_float(r[4 * j + 3]), ab)));
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              tma_store_2d(&tmap_d, smem_u32(buf), tile_n * BN + c, row0 + 16 * half);
              bulk_commit();
            }
          }
        }
      }
    }
    if (lane == 0) bulk_wait_all();
  }
  fence_before();
  __syncthreads();
  if (threadIdx.x == 0 && *abort_flag && status) *status = kStatusTimeout;
  if (warp == 1) {
    fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(G::TMEM_COLS) : "memory");
  }
}

// ===========================================================================
// 2-SM variant: a CTA pair (cluster of 2) computes a 256 x 256 tile with
// tcgen05.mma.cta_group::2 (M = 256, N = 256, K = 64).  Each CTA loads its own
// 128 rows of A and its own 128 rows of B, so per SM the operand traffic per
// FLOP is 2/3 of the single-CTA 128 x 256 tile; each CTA holds its 128 rows x
// 256 columns of the accumulator.  Scales: each CTA loads the scales of its A
// rows and of all 256 B rows (the MMA reads them from its own TMEM).
// Protocol (same shared-memory offsets in both CTAs):
//   full[s]    -- in the leader (rank 0) only: the leader's producer arms it
//                 with both CTAs' bytes; both CTAs' loads complete on it.
//   empty[s]   -- in both: the leader's MMA commit arrives on both.
//   acc_full   -- in both: the leader's commit at the end of a tile.
//   acc_empty  -- in the leader: 4 epilogue warps of each CTA arrive.
// ===========================================================================
constexpr int P_STAGE_A = 128 * BK_BYTES;        // own A rows
constexpr int P_STAGE_B = 128 * BK_BYTES;        // own B rows
constexpr int P_EPI_WARPS = 8;                   // two per TMEM lane quarter, 128 columns each
constexpr int P_THREADS = 64 + 32 * P_EPI_WARPS;
constexpr int P_OUT_STAGING = P_EPI_WARPS * 2048;
// Per-stage scale data: 512-byte atoms of 128 rows x 4 scale bytes.  NVFP4
// (16-element blocks) needs 4 atoms per 128 rows for a K = 256 stage, MXFP4
// (32-element blocks) 2.
template <bool MX>
struct PairCfg {
  static constexpr int ATOMS = MX ? 2 : KB_PER_STAGE;
  static constexpr int SFA = ATOMS * 512;       // own A rows' scales
  static constexpr int SFB = 2 * ATOMS * 512;   // all 256 B rows' scales
  static constexpr int STAGE = P_STAGE_A + P_STAGE_B + SFA + SFB;
  static constexpr int STAGES = (232448 - P_OUT_STAGING - 1024 - 512) / STAGE;
  static constexpr int SMEM = STAGES * STAGE + P_OUT_STAGING + 1024 + 512;
};
constexpr uint32_t P_SF_W = 4 + 8;               // SFA 4 + SFB (256 rows) 8 columns per K block
constexpr uint32_t P_SF_COL = 256;
constexpr uint32_t P_TMEM_COLS = 512;            // 256 accumulator + 2 x 4 K blocks x 12 scale columns
// M = 256 (>> 4 = 16 at bit 24), N = 256 (>> 3 = 32 at bit 17), E2M1 x E2M1, E4M3 scales
constexpr uint32_t P_IDESC = (1u << 7) | (1u << 10) | ((256u >> 3) << 17) | ((256u >> 4) << 24);
// MXFP4: the same with UE8M0 scales (bit 23); the scale-factor ids (bits
// 29-30 for A, 4-5 for B) are added per MMA.
constexpr uint32_t P_IDESC_MX = P_IDESC | (1u << 23);

// Optional NVFP4 quantization of the bf16 output rows in the epilogue (the
// next layer's rowwise input), with a provided tensor scale.
struct EpiQuant {
  uint8_t* codes;        // [M, N/2]
  uint8_t* scales;       // [M, N/16] row-major, or the GEMM scale layout
  const float* alpha;    // tensor scale of the output (device)
  uint32_t* amax;        // max |D| over the output (float bits), or null
  int gemm_layout;
  int write_d;           // also store D (bf16)
};

constexpr int kNoEpiQuant = -1;

// Byte offset of the scale of (row m, K-block j) in the GEMM scale layout
// (512-byte atoms of 128 rows x 4 K-blocks, K-atoms fastest).
__device__ __forceinline__ int64_t gemm_scale_byte(int64_t m, int64_t j, int64_t kblocks) {
  return ((m >> 7) * (kblocks >> 2) + (j >> 2)) * 512 + (m & 31) * 16 + ((m >> 5) & 3) * 4 + (j & 3);
}

// Tile order of the CTA-pair kernel: groups of `gm` M-tiles (the whole N
// range each), M fastest inside a group.  A wave of pairs then touches only
// one group's A panels and its B panels, which stay in L2 while the group is
// worked through, instead of every A panel per wave (the M-fastest order
// over the full M range re-read A from DRAM on the K = 14336 / 8192 shapes).
__device__ __forceinline__ void pair_tile_coords(int tile, int m_tiles, int n_tiles, int gm, int& tile_m,
                                                 int& tile_n) {
  const int group = tile / (gm * n_tiles);
  const int local = tile - group * gm * n_tiles;
  const int m0 = group * gm;
  const int rows = min(gm, m_tiles - m0);
  tile_m = m0 + local % rows;
  tile_n = local / rows;
}

// VS (vector scales): alpha_a holds one tensor scale per row of A ([M]) and
// alpha_b one per row of B ([N]); the epilogue scales D[m, n] by
// alpha_a[m] then alpha_b[n].
template <int QMODE, bool MX = false, bool VS = false>
__global__ void __launch_bounds__(P_THREADS, 1)
    nvfp4_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
                           const __grid_constant__ CUtensorMap tmap_d, const __grid_constant__ CUtensorMap tmap_sfa,
                           const __grid_constant__ CUtensorMap tmap_sfb, const float* __restrict__ alpha_a,
                           const float* __restrict__ alpha_b, int M, int N, int K, int out_fp32, int32_t* status,
                           const EpiQuant eq, int group_m) {
  pdl_entry();
  using PC = PairCfg<MX>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = sA + PC::STAGES * P_STAGE_A;
  uint8_t* sSFA = sB + PC::STAGES * P_STAGE_B;
  uint8_t* sSFB = sSFA + PC::STAGES * PC::SFA;
  uint8_t* sOut = sSFB + PC::STAGES * PC::SFB;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sOut + P_OUT_STAGING);
  uint64_t* full = bars;
  uint64_t* empty = bars + PC::STAGES;
  uint64_t* acc_full = bars + 2 * PC::STAGES;
  uint64_t* acc_empty = bars + 2 * PC::STAGES + 1;
  uint64_t* drain = bars + 2 * PC::STAGES + 2;   // tensor-op drain after an abort
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * PC::STAGES + 3);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int pair = static_cast<int>(blockIdx.x) >> 1, num_pairs = static_cast<int>(gridDim.x) >> 1;
  const int m_tiles = M / 256;
  const int num_tiles = m_tiles * (N / 256);
  const int kblocks64 = K / 64;
  const int katoms = MX ? K / 128 : K / 64;   // scale atoms along K per 128 rows
  const int kstages = (K + 255) / 256;

  if (threadIdx.x == 0) {
    for (int s = 0; s < PC::STAGES; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), 1);
    }
    mbar_init(smem_u32(acc_full), 1);
    mbar_init(smem_u32(acc_empty), 2 * P_EPI_WARPS);  // every epilogue warp of both CTAs
    mbar_init(smem_u32(drain), 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(P_TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  fence_before();
  __syncwarp();
  cluster_sync();  // barriers of both CTAs initialised, TMEM allocated
  fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ---------------- producer (both CTAs; one elected lane runs the loop) ----------------
    // The lane is elected once (elect.sync) and walks every stage alone;
    // nothing in the loop needs the rest of the warp.
    if (elect_one()) {
      int it = 0;
      bool stop = false;
      for (int tile = pair; tile < num_tiles && !stop; tile += num_pairs) {
        int tile_m, tile_n;
        pair_tile_coords(tile, m_tiles, N / 256, group_m, tile_m, tile_n);
        for (int kt = 0; kt < kstages; ++kt, ++it) {
          const int s = it % PC::STAGES;
          const uint32_t ph = (it / PC::STAGES) & 1;
          if (!mbar_wait(smem_u32(&empty[s]), ph ^ 1, abort_flag)) {
            stop = true;
            break;
          }
          const uint32_t fb_leader = map_to_rank(smem_u32(&full[s]), 0);
          const uint32_t dA = smem_u32(sA + s * P_STAGE_A), dB = smem_u32(sB + s * P_STAGE_B);
          const uint32_t dSA = smem_u32(sSFA + s * PC::SFA), dSB = smem_u32(sSFB + s * PC::SFB);
          // scale atoms viewed as rows of 256 bytes: a stage is 8 rows per 128 operand rows
          const int ysa = ((tile_m * 2 + static_cast<int>(rank)) * katoms + PC::ATOMS * kt) * 2;
          const int ysb = ((tile_n * 2) * katoms + PC::ATOMS * kt) * 2;
          if (leader) mbar_expect_tx(smem_u32(&full[s]), 2 * PC::STAGE);
          tma_load_2d_pair(dA, &tmap_a, kt * BK_BYTES, tile_m * 256 + 128 * rank, fb_leader);
          tma_load_2d_pair(dB, &tmap_b, kt * BK_BYTES, tile_n * 256 + 128 * rank, fb_leader);
          tma_load_2d_pair(dSA, &tmap_sfa, 0, ysa, fb_leader);
          tma_load_2d_pair(dSB, &tmap_sfb, 0, ysb, fb_leader);
          tma_load_2d_pair(dSB + PC::SFA, &tmap_sfb, 0, ysb + 2 * katoms, fb_leader);
        }
      }
      if (*abort_flag && leader) {
        // a wait gave up somewhere: let the copies already issued land
        // before the CTA exits (each wait again bounded)
        for (int i = (it > PC::STAGES ? it - PC::STAGES : 0); i < it; ++i) {
          const uint32_t bar = smem_u32(&full[i % PC::STAGES]), ph = (i / PC::STAGES) & 1;
          mbar_wait_bounded(bar, ph);
        }
      }
    }
  } else if (warp == 1) {
    if (leader && elect_one()) {
      // ---------------- MMA issuer (leader CTA, one elected lane) ----------------
      // Per stage: wait for its data, copy its scales into TMEM (one slot per
      // K block, two slot sets used alternately so the copies never overwrite
      // scales an earlier, still-running MMA reads), issue its MMAs, release
      // the stage.  The lane is elected once with elect.sync and runs the
      // whole loop.  Measured on B200 at 8192 x 14336 x 4096: about 12%
      // faster than the warp stepping through every stage together (a
      // reconvergence around each issue) and far faster than a plain lane-0
      // branch.
      const int my_tiles = (num_tiles - pair + num_pairs - 1) / num_pairs;
      const int total = my_tiles * kstages;
      // stage counters kept incrementally (no divisions on the issue path)
      int kt = 0, s = 0;
      uint32_t full_ph = 0, acc_ph = 0;
      for (int g = 0; g < total; ++g) {
        if (kt == 0) {
          // the epilogue must have drained the previous tile's accumulator
          if (!mbar_wait(smem_u32(acc_empty), acc_ph ^ 1, abort_flag)) break;
          acc_ph ^= 1;
          fence_after();
        }
        if (!mbar_wait(smem_u32(&full[s]), full_ph, abort_flag)) break;
        fence_after();
        const uint32_t sfa_s = smem_u32(sSFA + s * PC::SFA);
        const uint32_t sfb_s = smem_u32(sSFB + s * PC::SFB);
        const uint32_t set = static_cast<uint32_t>(g & 1) * KB_PER_STAGE;
        const int nk = min(KB_PER_STAGE, kblocks64 - KB_PER_STAGE * kt);
        const uint64_t adesc = desc_sw128(smem_u32(sA + s * P_STAGE_A));
        const uint64_t bdesc = desc_sw128(smem_u32(sB + s * P_STAGE_B));
        // NVFP4: each K block's scale atom is copied right before the MMA
        // that reads it, so copies and MMAs interleave on the tensor pipe
        // (measured on B200 about 12% faster than a stage's copies issued as
        // a group first: 8192 x 14336 x 4096 208 -> 185 us).  MXFP4 (one
        // atom per two MMAs, half the copies) measured faster with its
        // copies grouped (183 vs 197 us), so it keeps that order.
        if constexpr (MX) {
          for (int ka = 0; ka < (nk + 1) / 2; ++ka) {
            const uint32_t colc = tmem + P_SF_COL + (set + ka) * P_SF_W;
            tmem_cp_sf_pair(colc, desc_sf(sfa_s + 512 * ka));
            tmem_cp_sf_pair(colc + 4, desc_sf(sfb_s + 512 * ka));
            tmem_cp_sf_pair(colc + 8, desc_sf(sfb_s + PC::SFA + 512 * ka));
          }
        }
        for (int kk = 0; kk < nk; ++kk) {
          if constexpr (!MX) {
            const uint32_t colc = tmem + P_SF_COL + (set + kk) * P_SF_W;
            tmem_cp_sf_pair(colc, desc_sf(sfa_s + 512 * kk));
            tmem_cp_sf_pair(colc + 4, desc_sf(sfb_s + 512 * kk));
            tmem_cp_sf_pair(colc + 8, desc_sf(sfb_s + PC::SFA + 512 * kk));
          }
          const uint32_t acc = (kt > 0 || kk > 0) ? 1u : 0u;
          if constexpr (MX) {
            // MMA kk reads scale bytes 2 (kk & 1), +1 of atom kk / 2's columns
            const uint32_t col = tmem + P_SF_COL + (set + kk / 2) * P_SF_W;
            const uint32_t sf_id = 2u * static_cast<uint32_t>(kk & 1);
            mma_mxf4_pair(tmem, adesc + 2 * kk, bdesc + 2 * kk, P_IDESC_MX | (sf_id << 29) | (sf_id << 4), acc,
                          col, col + 4);
          } else {
            const uint32_t col = tmem + P_SF_COL + (set + kk) * P_SF_W;
            mma_mxf4nvf4_pair(tmem, adesc + 2 * kk, bdesc + 2 * kk, P_IDESC, acc, col, col + 4);
          }
        }
        umma_commit_pair(smem_u32(&empty[s]));
        if (kt == kstages - 1) umma_commit_pair(smem_u32(acc_full));
        if (++s == PC::STAGES) {
          s = 0;
          full_ph ^= 1;
        }
        if (++kt == kstages) kt = 0;
      }
      if (*abort_flag) {
        // a wait gave up: the copies and MMAs already issued (into both
        // CTAs' TMEM) may still run; let them finish (bounded) before the
        // pair frees TMEM
        umma_commit_pair(smem_u32(drain));
        mbar_wait_bounded(smem_u32(drain), 0);
      }
    }
  } else {
    // ---------------- epilogue (warps 2..9 of both CTAs) ----------------
    // Warp w reads TMEM lanes 32 (w % 4) .. + 31 and columns 128 h .. + 127
    // (h = 0 for warps 2-5, 1 for warps 6-9): two warps share each lane
    // quarter, each converting and storing half of the tile's columns.
    const int q = warp & 3, h = (warp - 2) >> 2;
    uint8_t* buf = sOut + (warp - 2) * 2048;
    // one factor for the whole product (MXFP4: no tensor scales), or per-row
    // and per-column factors (VS)
    const float ab = (MX || VS) ? 1.0f : __fmul_rn(__ldg(alpha_a), __ldg(alpha_b));
    const uint32_t acc_empty_leader = map_to_rank(smem_u32(acc_empty), 0);
    float eq_alpha = 0.0f, epi_amax = 0.0f;
    if constexpr (QMODE != kNoEpiQuant) eq_alpha = __ldg(eq.alpha);
    int ti = 0;
    for (int tile = pair; tile < num_tiles; tile += num_pairs, ++ti) {
      int tile_m, tile_n;
      pair_tile_coords(tile, m_tiles, N / 256, group_m, tile_m, tile_n);
      if (!mbar_wait(smem_u32(acc_full), ti & 1, abort_flag)) break;
      fence_after();
      const int row0 = tile_m * 256 + 128 * static_cast<int>(rank) + 32 * q;
      const int col0 = tile_n * 256 + 128 * h;
      const uint32_t taddr = tmem + (static_cast<uint32_t>(32 * q) << 16) + 128 * h;
      // VS: D = RN(RN(acc * alpha_a[m]) * alpha_b[n])
      const float am = VS ? __ldg(alpha_a + row0 + lane) : 1.0f;
      auto scale = [&](uint32_t acc_bits, int col) -> float {
        if constexpr (VS) return __fmul_rn(__fmul_rn(__uint_as_float(acc_bits), am), __ldg(alpha_b + col0 + col));
        return __fmul_rn(__uint_as_float(acc_bits), ab);
      };
      // two adjacent columns as packed bf16 (one packed multiply without VS)
      auto scale_bf16x2 = [&](uint32_t acc0, uint32_t acc1, int col) -> uint32_t {
        __nv_bfloat162 b2;
        if constexpr (VS) {
          b2 = __floats2bfloat162_rn(scale(acc0, col), scale(acc1, col + 1));
        } else {
          const float2 p = __fmul2_rn(make_float2(__uint_as_float(acc0), __uint_as_float(acc1)), make_float2(ab, ab));
          b2 = __floats2bfloat162_rn(p.x, p.y);
        }
        return *reinterpret_cast<const uint32_t*>(&b2);
      };
      if (!out_fp32) {
        // two rounds of 64 columns: load, wait, convert to packed bf16; the
        // accumulator is handed back once the whole row is in registers
        // (measured faster than loading all 128 columns before one wait)
        uint32_t packed[64];
#pragma unroll
        for (int c = 0; c < 128; c += 64) {
          uint32_t r[64];
          tmem_ld32_nowait(taddr + c, r);
          tmem_ld32_nowait(taddr + c + 32, r + 32);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 32; ++j) packed[c / 2 + j] = scale_bf16x2(r[2 * j], r[2 * j + 1], c + 2 * j);
        }
        fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(acc_empty_leader);
        if constexpr (QMODE != kNoEpiQuant) {
          // this lane's output row, 8 blocks of 16 columns, two at a time,
          // from the bf16 values just formed (exact in fp32)
          const int64_t grow = row0 + lane;
#pragma unroll
          for (int jb = 0; jb < 8; jb += 2) {
            float2 v[16];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const uint32_t wa = packed[8 * jb + e], wb = packed[8 * jb + 8 + e];
              v[2 * e] = make_float2(__uint_as_float(wa << 16), __uint_as_float(wb << 16));
              v[2 * e + 1] = make_float2(__uint_as_float(wa & 0xFFFF0000u), __uint_as_float(wb & 0xFFFF0000u));
            }
#pragma unroll
            for (int i = 0; i < 16; ++i) epi_amax = fmaxf(epi_amax, fmaxf(fabsf(v[i].x), fabsf(v[i].y)));
            Packed16 pa, pb;
            uint32_t sa, sb;
            quantize_pair_rne<QMODE == kModeFourSix>(v, eq_alpha, pa, pb, sa, sb);
            const int64_t gcb = (col0 + 16 * jb) / 16;
            *reinterpret_cast<uint4*>(eq.codes + grow * (N / 2) + 8 * gcb) = make_uint4(pa.lo, pa.hi, pb.lo, pb.hi);
            if (eq.gemm_layout) {
              eq.scales[gemm_scale_byte(grow, gcb, N / 16)] = static_cast<uint8_t>(sa);
              eq.scales[gemm_scale_byte(grow, gcb + 1, N / 16)] = static_cast<uint8_t>(sb);
            } else {
              eq.scales[grow * (N / 16) + gcb] = static_cast<uint8_t>(sa);
              eq.scales[grow * (N / 16) + gcb + 1] = static_cast<uint8_t>(sb);
            }
          }
          if (!eq.write_d) continue;
        }
#pragma unroll
        for (int p = 0; p < 2; ++p) {        // 64-column pieces
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            if (lane == 0) bulk_wait_read<0>();
            __syncwarp();
            if ((lane >> 4) == half) {
              uint8_t* rowp = buf + (lane & 15) * 128;
#pragma unroll
              for (int j = 0; j < 8; ++j)
                *reinterpret_cast<uint4*>(rowp + ((j ^ (lane & 7)) << 4)) =
                    make_uint4(packed[32 * p + 4 * j], packed[32 * p + 4 * j + 1], packed[32 * p + 4 * j + 2],
                               packed[32 * p + 4 * j + 3]);
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              tma_store_2d(&tmap_d, smem_u32(buf), col0 + 64 * p, row0 + 16 * half);
              bulk_commit();
            }
          }
        }
      } else {
#pragma unroll 1
        for (int c = 0; c < 128; c += 32) {
          uint32_t r[32];
          tmem_ld32_nowait(taddr + c, r);
          tmem_ld_wait();
          if (c + 32 == 128) {
            fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(acc_empty_leader);
          }
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            if (lane == 0) bulk_wait_read<0>();
            __syncwarp();
            if ((lane >> 4) == half) {
              uint8_t* rowp = buf + (lane & 15) * 128;
#pragma unroll
              for (int j = 0; j < 8; ++j)
                *reinterpret_cast<uint4*>(rowp + ((j ^ (lane & 7)) << 4)) =
                    make_uint4(__float_as_uint(scale(r[4 * j], c + 4 * j)),
                               __float_as_uint(scale(r[4 * j + 1], c + 4 * j + 1)),
                               __float_as_uint(scale(r[4 * j + 2], c + 4 * j + 2)),
                               __float_as_uint(scale(r[4 * j + 3], c + 4 * j + 3)));
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              tma_store_2d(&tmap_d, smem_u32(buf), col0 + c, row0 + 16 * half);
              bulk_commit();
            }
          }
        }
      }
    }
    if (lane == 0) bulk_wait_all();
    if constexpr (QMODE != kNoEpiQuant) {
      if (eq.amax) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) epi_amax = fmaxf(epi_amax, __shfl_xor_sync(0xFFFFFFFFu, epi_amax, o));
        if (lane == 0) atomicMax(eq.amax, __float_as_uint(epi_amax));
      }
    }
  }
  fence_before();
  __syncwarp();
  // neither CTA may leave (or free TMEM) while its peer can still touch its
  // shared memory or its TMEM
  cluster_sync();
  if (threadIdx.x == 0 && *abort_flag && status) *status = kStatusTimeout;
  if (warp == 1) {
    fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(P_TMEM_COLS) : "memory");
  }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 2D map over packed codes [rows, K/2] bytes, box 128 B x box_rows, 128-byte swizzle.
bool make_map(CUtensorMap* map, const void* base, int64_t rows, int64_t kbytes, int box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(kbytes), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(kbytes)};
  const cuuint32_t box[2] = {BK_BYTES, static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2D map over the output D [M, N] (row stride ldd elements): boxes of 16 rows
// x 128 bytes (64 bf16 or 32 fp32 columns), 128-byte swizzle, for TMA stores.
bool make_out_map(CUtensorMap* map, void* base, int64_t M, int64_t N, int64_t ldd, bool fp32) {
  auto fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t esize = fp32 ? 4 : 2;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(M)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(ldd) * esize};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(128 / esize), 16};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, fp32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides,
            box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int BN>
cudaError_t launch(const uint8_t* A, const uint8_t* sA, const float* alphaA, const uint8_t* B, const uint8_t* sB,
                   const float* alphaB, int64_t M, int64_t N, int64_t K, void* D, int out_dtype, int64_t ldd,
                   int32_t* status, cudaStream_t st) {
  using G = Cfg<BN>;
  const bool fp32 = out_dtype == NVFP4_OUT_DTYPE_FP32;
  CUtensorMap ma, mb, md;
  if (!make_map(&ma, A, M, K / 2, BM) || !make_map(&mb, B, N, K / 2, BN) || !make_out_map(&md, D, M, N, ldd, fp32))
    return cudaErrorInvalidValue;
  static bool attr_set[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(nvfp4_gemm_kernel<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize, G::SMEM);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  const int64_t tiles = (M / BM) * (N / BN);
  const int grid = static_cast<int>(tiles < sm_count() ? tiles : sm_count());  // persistent: one CTA per SM
  launch_k(nvfp4_gemm_kernel<BN>, dim3(grid), dim3(NUM_THREADS), G::SMEM, st, 1u, ma, mb, md, sA, sB, alphaA, alphaB, static_cast<int>(M),
                                                            static_cast<int>(N), static_cast<int>(K), fp32, status);
  note_launch();
  return cudaGetLastError();
}

// Scale array of an operand (GEMM layout) viewed as rows of 256 bytes:
// 512-byte atoms -> two rows each; one stage of 4 atoms (NVFP4) = 8 rows, of
// 2 atoms (MXFP4, one atom per 128 K) = 4 rows.
bool make_sf_map(CUtensorMap* map, const void* base, int64_t rows, int64_t K, bool mx = false) {
  auto fn = encode_fn();
  if (!fn) return false;
  const int64_t bytes = (rows / 128) * (mx ? K / 128 : K / 64) * 512;
  const cuuint64_t dims[2] = {256, static_cast<cuuint64_t>(bytes / 256)};
  const cuuint64_t strides[1] = {256};
  const cuuint32_t box[2] = {256, mx ? 4u : 8u};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int QMODE, bool MX = false, bool VS = false>
cudaError_t launch_pair(const uint8_t* A, const uint8_t* sA, const float* alphaA, const uint8_t* B, const uint8_t* sB,
                        const float* alphaB, int64_t M, int64_t N, int64_t K, void* D, int out_dtype, int64_t ldd,
                        int32_t* status, const EpiQuant& eq, cudaStream_t st) {
  const bool fp32 = out_dtype == NVFP4_OUT_DTYPE_FP32;
  CUtensorMap ma, mb, md, msa, msb;
  std::memset(&md, 0, sizeof(md));   // unused when the epilogue writes no D
  if (!make_map(&ma, A, M, K / 2, 128) || !make_map(&mb, B, N, K / 2, 128) || !make_sf_map(&msa, sA, M, K, MX) ||
      !make_sf_map(&msb, sB, N, K, MX))
    return cudaErrorInvalidValue;
  if (D && !make_out_map(&md, D, M, N, ldd, fp32)) return cudaErrorInvalidValue;
  static bool attr_set[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_set[dev]) {
    cudaError_t e =
        cudaFuncSetAttribute(nvfp4_gemm_pair_kernel<QMODE, MX, VS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             PairCfg<MX>::SMEM);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  if (QMODE != kNoEpiQuant && eq.amax) {
    cudaError_t e = cudaMemsetAsync(eq.amax, 0, sizeof(uint32_t), st);
    if (e != cudaSuccess) return e;
  }
  const int64_t tiles = (M / 256) * (N / 256);
  const int64_t pairs = tiles < sm_count() / 2 ? tiles : sm_count() / 2;  // persistent: one pair per TPC
  // M-tiles per raster group: as many as keep the group's A panels plus all
  // of B within about 64 MB of L2 (operand bytes per 256-row panel: K / 2
  // codes + K / 16 scales)
  const int64_t panel = 256 * (K / 2 + K / 16);
  const int64_t m_tiles = M / 256, n_tiles = N / 256;
  int64_t gm = (int64_t(64) << 20) / panel - n_tiles;
  gm = gm < 1 ? 1 : (gm > m_tiles ? m_tiles : gm);
  cudaError_t e = launch_k(nvfp4_gemm_pair_kernel<QMODE, MX, VS>, dim3(static_cast<unsigned>(2 * pairs)),
                           dim3(P_THREADS), PairCfg<MX>::SMEM, st, 2u, ma, mb, md, msa, msb, alphaA, alphaB,
                           static_cast<int>(M), static_cast<int>(N), static_cast<int>(K), static_cast<int>(fp32),
                           status, eq, static_cast<int>(gm));
  note_launch();
  return e;
}

}  // namespace

cudaError_t gemm_launch(const uint8_t* A, const uint8_t* sA, const float* alphaA, const uint8_t* B, const uint8_t* sB,
                        const float* alphaB, int64_t M, int64_t N, int64_t K, void* D, int out_dtype, int64_t ldd,
                        int32_t* status, cudaStream_t st) {
  if (M % 256 == 0 && N % 256 == 0) {
    const EpiQuant none{nullptr, nullptr, nullptr, nullptr, 0, 1};
    return launch_pair<kNoEpiQuant>(A, sA, alphaA, B, sB, alphaB, M, N, K, D, out_dtype, ldd, status, none, st);
  }
  if (N % 256 == 0) return launch<256>(A, sA, alphaA, B, sB, alphaB, M, N, K, D, out_dtype, ldd, status, st);
  return launch<128>(A, sA, alphaA, B, sB, alphaB, M, N, K, D, out_dtype, ldd, status, st);
}

cudaError_t gemm_vs_launch(const uint8_t* A, const uint8_t* sA, const float* alphaA, const uint8_t* B,
                           const uint8_t* sB, const float* alphaB, int64_t M, int64_t N, int64_t K, void* D,
                           int out_dtype, int64_t ldd, int32_t* status, cudaStream_t st) {
  const EpiQuant none{nullptr, nullptr, nullptr, nullptr, 0, 1};
  return launch_pair<kNoEpiQuant, false, true>(A, sA, alphaA, B, sB, alphaB, M, N, K, D, out_dtype, ldd, status,
                                               none, st);
}

cudaError_t mx_gemm_launch(const uint8_t* A, const uint8_t* sA, const uint8_t* B, const uint8_t* sB, int64_t M,
                           int64_t N, int64_t K, void* D, int out_dtype, int64_t ldd, int32_t* status, cudaStream_t st) {
  const EpiQuant none{nullptr, nullptr, nullptr, nullptr, 0, 1};
  return launch_pair<kNoEpiQuant, true>(A, sA, nullptr, B, sB, nullptr, M, N, K, D, out_dtype, ldd, status, none, st);
}

cudaError_t gemm_quantize_launch(const uint8_t* A, const uint8_t* sA, const float* alphaA, const uint8_t* B,
                                 const uint8_t* sB, const float* alphaB, int64_t M, int64_t N, int64_t K, void* D,
                                 int64_t ldd, int mode, bool gemm_layout, const float* alpha_out, uint8_t* codes,
                                 uint8_t* scales, float* amax_out, int32_t* status, cudaStream_t st) {
  const EpiQuant eq{codes, scales, alpha_out, reinterpret_cast<uint32_t*>(amax_out), gemm_layout ? 1 : 0,
                    D ? 1 : 0};
  if (mode == kModeFourSix)
    return launch_pair<kModeFourSix>(A, sA, alphaA, B, sB, alphaB, M, N, K, D, NVFP4_OUT_DTYPE_BF16, ldd, status,
                                     eq, st);
  return launch_pair<kModeRTN>(A, sA, alphaA, B, sB, alphaB, M, N, K, D, NVFP4_OUT_DTYPE_BF16, ldd, status, eq, st);
}

}  // namespace nvfp4
