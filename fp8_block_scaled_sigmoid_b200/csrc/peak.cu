// FP8 tensor-core peak of this GPU, measured: a loop of tcgen05 MMAs that
// touches no global memory.
//
// The roofline of the expert GEMMs needs the dense FP8 rate of the part it
// runs on, at the clocks it actually holds.  Each CTA (one per SM) fills a
// 128x128 E4M3 A tile and a 256x128 E4M3 B tile in shared memory once, then
// one thread issues `iters` K blocks of four 128x256x32 MMAs into a 256-column
// TMEM accumulator (two accumulators alternate, as the GEMMs' ping-pong
// does).  With `block_scaled` the MMAs are kind::mxf8f6f4.block_scale with
// unit (2^0) UE8M0 scale factors in TMEM, the instruction the power-of-two
// GEMM issues; otherwise kind::f8f6f4, the promoting GEMM's instruction.
// FLOPs per launch = ctas * iters * 4 * 2*128*256*32.
//
// The operand bytes are a fixed pseudo-random pattern with no NaN codes, so
// the multipliers toggle as they do on real data (power, hence clocks, depend
// on it).
#include "moe_common.cuh"

namespace moe {
namespace {

constexpr int kPM = 128, kPN = 256, kPK = 128;
constexpr int kPA = kPM * kPK, kPB = kPN * kPK;  // bytes of the A and B tiles
// 1024 alignment slack + A + B + three 512-byte scale atoms + barrier; the
// launch asks for more than half an SM's shared memory so that one CTA runs
// per SM and the TMEM allocation never waits on a co-resident CTA.
constexpr int kPeakSmem = 120 * 1024;

__global__ void __launch_bounds__(128, 1) fp8_mma_peak_kernel(int iters, int block_scaled,
                                                              float* sink, int32_t* dev_err) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* base = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint8_t* sA = base;
  uint8_t* sB = base + kPA;
  uint8_t* sf = sB + kPB;                                   // 3 x 512 bytes of exponents
  uint64_t* bar = reinterpret_cast<uint64_t*>(sf + 1536);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar + 1);
  const int tid = threadIdx.x, warp = tid >> 5;

  // operand pattern: sign and low exponent/mantissa bits from a hash of the
  // byte index and the CTA, exponent field <= 7 (no NaN 0x7F/0xFF codes)
  uint32_t* a32 = reinterpret_cast<uint32_t*>(sA);
  for (int i = tid; i < (kPA + kPB) / 4; i += blockDim.x) {
    uint32_t h = (static_cast<uint32_t>(i) + 0x9E3779B9u * (blockIdx.x + 1)) * 0x85EBCA6Bu;
    h ^= h >> 13;
    h *= 0xC2B2AE35u;
    h ^= h >> 16;
    a32[i] = h & 0xBFBFBFBFu;  // clear bit 6 of every byte: exponent field < 8
  }
  uint32_t* sf32 = reinterpret_cast<uint32_t*>(sf);
  for (int i = tid; i < 1536 / 4; i += blockDim.x) sf32[i] = 0x7F7F7F7Fu;  // 2^0
  if (tid == 0) {
    mbar_init(bar, 1);
    fence_barrier_init();
  }
  fence_proxy_async_smem();
  if (warp == 0) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // The scale factors live in columns the accumulators do not use: with two
  // 256-column accumulators there are none, so the block-scaled loop keeps one
  // accumulator (columns 0..255) and its scale factors at 256..271.
  if (tid == 0) {
    const uint64_t ad = smem_desc_sw128(smem_u32(sA));
    const uint64_t bd = smem_desc_sw128(smem_u32(sB));
    if (block_scaled) {
      const uint32_t sfs = smem_u32(sf);
      const uint32_t t_sfa = tmem + 256, t_sfb = tmem + 264;
      tmem_cp_32x128b_x4(t_sfa, smem_desc_interleave(sfs, 128));
      tmem_cp_32x128b_x4(t_sfb, smem_desc_interleave(sfs + 512, 128));
      tmem_cp_32x128b_x4(t_sfb + 4, smem_desc_interleave(sfs + 1024, 128));
      for (int it = 0; it < iters; ++it) {
        const uint32_t idesc = instr_desc_mx(kPM, kPN, static_cast<uint32_t>(it & 3));
#pragma unroll
        for (int k = 0; k < kPK / 32; ++k)
          mma_mxf8f6f4(tmem, ad + 2 * k, bd + 2 * k, idesc, (it > 0 || k > 0) ? 1u : 0u, t_sfa,
                       t_sfb);
      }
    } else {
      const uint32_t idesc = instr_desc(kFmtE4M3, kFmtE4M3, kPM, kPN);
      for (int it = 0; it < iters; ++it) {
        const uint32_t dt = tmem + static_cast<uint32_t>((it & 1) * kPN);
#pragma unroll
        for (int k = 0; k < kPK / 32; ++k)
          mma_f8f6f4(dt, ad + 2 * k, bd + 2 * k, idesc, (it > 1 || k > 0) ? 1u : 0u);
      }
    }
    mma_commit(bar);
  }
  __syncwarp();
  // every thread waits for the MMAs (bounded), then warp 0 reads one column
  const bool ok = mbar_wait(bar, 0, nullptr, dev_err);
  tc_fence_after();
  if (warp == 0) {
    float v[16];
    tmem_ld16(tmem, v);
    tmem_ld_wait();
    if (tid == 0 && sink) sink[blockIdx.x] = ok ? v[0] : 0.f;
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 512);
}

}  // namespace
}  // namespace moe

extern "C" moe_status moe_fp8_mma_peak(int block_scaled, int iters, int ctas, float* sink,
                                       int32_t* dev_err, moe_stream_t stream) {
  using namespace moe;
  if (iters < 1 || ctas < 1 || !sink) return MOE_ERR_INVALID_ARG;
  if (iters > (1 << 21) || ctas > 65535) return MOE_ERR_UNSUPPORTED;
  if (cudaFuncSetAttribute(fp8_mma_peak_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           kPeakSmem) != cudaSuccess)
    return MOE_ERR_CUDA;
  fp8_mma_peak_kernel<<<ctas, 128, kPeakSmem, static_cast<cudaStream_t>(stream)>>>(
      iters, block_scaled ? 1 : 0, sink, dev_err);
  MOE_CUDA_CHECK_LAUNCH();
  return MOE_OK;
}
