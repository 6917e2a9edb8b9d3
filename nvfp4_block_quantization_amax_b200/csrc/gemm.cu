// gemm.cu -- block-scaled NVFP4 GEMM on the sm_100a tensor cores.
//
//   D[m, n] = alphaA * alphaB * sum_k (qA[m,k] DeltaA[m,k/16]) (qB[n,k] DeltaB[n,k/16])
//
// The NVFP4 pretraining write-up (§四) describes the Blackwell tensor cores
// that read narrow values plus 8-bit block scales and accumulate in FP32; this
// kernel drives them directly:
//   * warp 0 (one lane): TMA producer.  Per K-stage of 256 elements it loads
//     the A tile (128 rows x 128 B) and the B tile (BN rows x 128 B) with 128-
//     byte swizzle, and the matching scale atoms (512 B per 128 rows x 64 K)
//     with bulk copies, into a ring of shared-memory stages guarded by
//     mbarriers.
//   * warp 1: allocates tensor memory; one lane copies each stage's scales
//     into TMEM (tcgen05.cp 32x128b.warpx4) and issues four
//     tcgen05.mma.kind::mxf4nvf4.block_scale.block16 (M=128, N=BN, K=64),
//     accumulating in TMEM, then commits the stage back to the producer.
//   * warps 2-5: epilogue.  Each reads its 32-lane quarter of the FP32
//     accumulator with tcgen05.ld, multiplies by alphaA * alphaB, converts to
//     bf16 (or keeps fp32) and stores.
// Every wait is bounded (about two seconds of %globaltimer); a wait that
// gives up raises an abort flag that every role checks, the kernel records
// NVFP4_ERR_TIMEOUT in the optional status word and still frees its TMEM.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cstdint>
#include <mutex>

#include "nvfp4_internal.h"

namespace nvfp4 {
namespace {

constexpr int BM = 128;
constexpr int BK_BYTES = 128;  // 256 FP4 values per row per stage
constexpr int STAGES = 4;
constexpr int NUM_THREADS = 192;
constexpr uint64_t kTimeoutNs = 2000000000ull;

template <int BN>
struct Cfg {
  static constexpr int A_STAGE = BM * BK_BYTES;
  static constexpr int B_STAGE = BN * BK_BYTES;
  static constexpr int SFA_STAGE = 4 * 512;
  static constexpr int SFB_STAGE = (BN / 128) * 4 * 512;
  static constexpr int STAGE = A_STAGE + B_STAGE + SFA_STAGE + SFB_STAGE;
  static constexpr int SMEM = STAGES * STAGE + 1024 /* alignment */ + 256 /* barriers */;
  static constexpr uint32_t TMEM_COLS = (BN + 16 + 4 * 4 * (BN / 128)) <= 256 ? 256 : 512;
  static constexpr uint32_t SFA_COL = BN;            // 4 columns per MMA k-block
  static constexpr uint32_t SFB_COL = BN + 16;       // 4 * (BN/128) columns per MMA k-block
  // Instruction descriptor (kind::mxf4nvf4): A and B are E2M1 (format 1),
  // K-major, scales E4M3, N >> 3 at bit 17, M >> 4 at bit 24.
  static constexpr uint32_t IDESC = (1u << 7) | (1u << 10) | ((uint32_t(BN) >> 3) << 17) | ((uint32_t(BM) >> 4) << 24);
};

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
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
// 8-row groups, descriptor version 1, layout SWIZZLE_128B (2) in bits 61-63.
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

// 32 lanes x 32 columns of 32-bit accumulators: thread t gets lane t's row.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]),
        "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

template <int BN>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    nvfp4_gemm_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
                      const uint8_t* __restrict__ sfa, const uint8_t* __restrict__ sfb,
                      const float* __restrict__ alpha_a, const float* __restrict__ alpha_b, void* __restrict__ d,
                      int64_t ldd, int M, int N, int K, int out_fp32, int32_t* status) {
  using G = Cfg<BN>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = sA + STAGES * G::A_STAGE;
  uint8_t* sSFA = sB + STAGES * G::B_STAGE;
  uint8_t* sSFB = sSFA + STAGES * G::SFA_STAGE;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sSFB + STAGES * G::SFB_STAGE);
  uint64_t* full = bars;
  uint64_t* empty = bars + STAGES;
  uint64_t* acc_full = bars + 2 * STAGES;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * STAGES + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m_tiles = M / BM;
  const int tile_m = blockIdx.x % m_tiles, tile_n = blockIdx.x / m_tiles;
  const int kblocks64 = K / 64;           // scale atoms along K
  const int kstages = (K + 255) / 256;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), 1);
    }
    mbar_init(smem_u32(acc_full), 1);
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
    if (lane == 0) {
      // ---------------- producer ----------------
      int issued = 0;
      for (int kt = 0; kt < kstages; ++kt) {
        const int s = kt % STAGES;
        const uint32_t ph = (kt / STAGES) & 1;
        if (!mbar_wait(smem_u32(&empty[s]), ph ^ 1, abort_flag)) break;
        ++issued;
        const int nk = min(4, kblocks64 - 4 * kt);  // 64-wide K blocks in this stage
        const uint32_t bytes = G::A_STAGE + G::B_STAGE + nk * 512 * (1 + BN / 128);
        const uint32_t fb = smem_u32(&full[s]);
        mbar_expect_tx(fb, bytes);
        tma_load_2d(smem_u32(sA + s * G::A_STAGE), &tmap_a, kt * BK_BYTES, tile_m * BM, fb);
        tma_load_2d(smem_u32(sB + s * G::B_STAGE), &tmap_b, kt * BK_BYTES, tile_n * BN, fb);
        bulk_load(smem_u32(sSFA + s * G::SFA_STAGE),
                  sfa + (static_cast<int64_t>(tile_m) * kblocks64 + 4 * kt) * 512, nk * 512, fb);
#pragma unroll
        for (int g = 0; g < BN / 128; ++g)
          bulk_load(smem_u32(sSFB + s * G::SFB_STAGE + g * 2048),
                    sfb + (static_cast<int64_t>(tile_n * (BN / 128) + g) * kblocks64 + 4 * kt) * 512, nk * 512, fb);
      }
      if (*abort_flag) {
        // A wait gave up somewhere: let the copies this thread issued land
        // before the CTA exits (each wait again bounded).
        for (int kt = (issued > STAGES ? issued - STAGES : 0); kt < issued; ++kt) {
          const uint32_t bar = smem_u32(&full[kt % STAGES]), ph = (kt / STAGES) & 1;
          const uint64_t t0 = globaltimer();
          while (!mbar_try_wait(bar, ph) && globaltimer() - t0 < kTimeoutNs) {
          }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer ----------------
      for (int kt = 0; kt < kstages; ++kt) {
        const int s = kt % STAGES;
        const uint32_t ph = (kt / STAGES) & 1;
        if (!mbar_wait(smem_u32(&full[s]), ph, abort_flag)) break;
        fence_after();
        const int nk = min(4, kblocks64 - 4 * kt);
        const uint32_t sfa_s = smem_u32(sSFA + s * G::SFA_STAGE);
        const uint32_t sfb_s = smem_u32(sSFB + s * G::SFB_STAGE);
        for (int kk = 0; kk < nk; ++kk) {
          tmem_cp_sf(tmem + G::SFA_COL + 4 * kk, desc_sf(sfa_s + 512 * kk));
#pragma unroll
          for (int g = 0; g < BN / 128; ++g)
            tmem_cp_sf(tmem + G::SFB_COL + 4 * (BN / 128) * kk + 4 * g, desc_sf(sfb_s + g * 2048 + 512 * kk));
        }
        const uint64_t adesc = desc_sw128(smem_u32(sA + s * G::A_STAGE));
        const uint64_t bdesc = desc_sw128(smem_u32(sB + s * G::B_STAGE));
        for (int kk = 0; kk < nk; ++kk) {
          // K = 64 FP4 values = 32 bytes: advance the start address by 2 x 16 B
          mma_mxf4nvf4(tmem, adesc + 2 * kk, bdesc + 2 * kk, G::IDESC, (kt > 0 || kk > 0) ? 1u : 0u,
                       tmem + G::SFA_COL + 4 * kk, tmem + G::SFB_COL + 4 * (BN / 128) * kk);
        }
        umma_commit(smem_u32(&empty[s]));
      }
      umma_commit(smem_u32(acc_full));
    }
  } else {
    // ---------------- epilogue (warps 2..5) ----------------
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    const bool ok = mbar_wait(smem_u32(acc_full), 0, abort_flag);
    fence_after();
    if (ok && !*abort_flag) {
      const float ab = __fmul_rn(__ldg(alpha_a), __ldg(alpha_b));
      const int64_t row = static_cast<int64_t>(tile_m) * BM + 32 * q + lane;
      const int64_t col0 = static_cast<int64_t>(tile_n) * BN;
#pragma unroll 1
      for (int c = 0; c < BN; c += 32) {
        uint32_t r[32];
        tmem_ld32(tmem + (static_cast<uint32_t>(32 * q) << 16) + c, r);
        if (out_fp32) {
          float4* dst = reinterpret_cast<float4*>(static_cast<float*>(d) + row * ldd + col0 + c);
#pragma unroll
          for (int j = 0; j < 8; ++j)
            dst[j] = make_float4(__fmul_rn(__uint_as_float(r[4 * j]), ab), __fmul_rn(__uint_as_float(r[4 * j + 1]), ab),
                                 __fmul_rn(__uint_as_float(r[4 * j + 2]), ab),
                                 __fmul_rn(__uint_as_float(r[4 * j + 3]), ab));
        } else {
          uint32_t w[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const __nv_bfloat162 h = __floats2bfloat162_rn(__fmul_rn(__uint_as_float(r[2 * j]), ab),
                                                           __fmul_rn(__uint_as_float(r[2 * j + 1]), ab));
            w[j] = *reinterpret_cast<const uint32_t*>(&h);
          }
          uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(d) + row * ldd + col0 + c);
#pragma unroll
          for (int j = 0; j < 4; ++j) dst[j] = make_uint4(w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
        }
      }
    }
  }
  fence_before();
  __syncthreads();
  if (threadIdx.x == 0 && *abort_flag && status) *status = kStatusTimeout;
  if (warp == 1) {
    fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(G::TMEM_COLS) : "memory");
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

template <int BN>
cudaError_t launch(const uint8_t* A, const uint8_t* sA, const float* alphaA, const uint8_t* B, const uint8_t* sB,
                   const float* alphaB, int64_t M, int64_t N, int64_t K, void* D, int out_dtype, int64_t ldd,
                   int32_t* status, cudaStream_t st) {
  using G = Cfg<BN>;
  CUtensorMap ma, mb;
  if (!make_map(&ma, A, M, K / 2, BM) || !make_map(&mb, B, N, K / 2, BN)) return cudaErrorInvalidValue;
  static bool attr_set[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(nvfp4_gemm_kernel<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize, G::SMEM);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  const int grid = static_cast<int>((M / BM) * (N / BN));
  nvfp4_gemm_kernel<BN><<<grid, NUM_THREADS, G::SMEM, st>>>(ma, mb, sA, sB, alphaA, alphaB, D, ldd,
                                                            static_cast<int>(M), static_cast<int>(N),
                                                            static_cast<int>(K), out_dtype == NVFP4_OUT_DTYPE_FP32,
                                                            status);
  note_launch();
  return cudaGetLastError();
}

}  // namespace

cudaError_t gemm_launch(const uint8_t* A, const uint8_t* sA, const float* alphaA, const uint8_t* B, const uint8_t* sB,
                        const float* alphaB, int64_t M, int64_t N, int64_t K, void* D, int out_dtype, int64_t ldd,
                        int32_t* status, cudaStream_t st) {
  if (N % 256 == 0) return launch<256>(A, sA, alphaA, B, sB, alphaB, M, N, K, D, out_dtype, ldd, status, st);
  return launch<128>(A, sA, alphaA, B, sB, alphaB, M, N, K, D, out_dtype, ldd, status, st);
}

}  // namespace nvfp4
