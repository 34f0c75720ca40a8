// Device-side building blocks for the replay decode kernels (sm_100a):
// mbarrier and bulk-copy (TMA) wrappers written as inline PTX, bounded waits that
// report a timeout through the status word instead of trapping, segment reductions
// over the lanes that share one state row, and FP8 e4m3 / BF16 conversions.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <stdint.h>

namespace replay {

constexpr int kGroupGemvWarps = 4;               // per consumer group: warps that stream the state rows
constexpr int kGroupWarps = kGroupGemvWarps + 1; // ... plus one warp for the decay weights and k . q
constexpr int kGroups = 2;                       // consumer groups per CTA
constexpr int kConsumerWarps = kGroups * kGroupWarps;
constexpr int kProducerWarps = 1;                // the warp that fills stages, in unit order
constexpr int kThreads = (kConsumerWarps + kProducerWarps) * 32;
constexpr int kMaxPos = 8;                       // query positions per verify call
constexpr int kMaxWindow = 32;                   // largest L (decay scans use one warp)
constexpr int kMaxStages = 8;
constexpr int kMaxChunkHeads = 8;                // heads of one k/q group a CTA takes in a row
constexpr int kUnitsPerIssue = 2;                // units whose copies share one bulk-copy instruction
constexpr int kRowsPerThread = 16;               // state rows one thread covers per row group
constexpr int kHeaderBytes = 256;                // the mbarriers and flags at the start of shared memory
// State rows of one row group: kGroupGemvWarps warps, 128/N rows per warp pass (a row of
// N floats takes N/4 lanes), kRowsPerThread rows per lane. A unit covers one row group of
// a head (or the whole head when it has fewer rows), so that every unit's tile is at most
// 32 KiB of FP32 and as many stages fit in shared memory whatever the head's P.
constexpr int row_group_rows(int N) { return kGroupGemvWarps * (128 / N) * kRowsPerThread; }
constexpr long long kWaitLimitCycles = 4000000000LL;  // ~2 s at the boost clock

// status word bits (device-detected errors; the host reads them with replay_check_status)
constexpr int32_t kErrWaitTimeout = 1 << 0;   // an mbarrier wait gave up
constexpr int32_t kErrPointer = 1 << 1;       // a buffer pointer word was out of range
constexpr int32_t kErrRollback = 1 << 2;      // n_keep outside [0, n_pos]
constexpr int32_t kErrSnapshot = 1 << 3;      // an imported snapshot does not match the layer (skipped)

// snapshot block of one sequence: a header of kSnapHeaderBytes (int32: magic, count, H, P,
// N, L, record bytes, 0), then the FP32 state [H][P][N], then [H][L] ring records
constexpr int kSnapHeaderBytes = 64;
constexpr int32_t kSnapMagic = 0x4E535052;  // "RPSN"

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
// Tests the phase with the given parity; if it is not complete the thread is suspended
// in hardware (no issue slots used) until it completes or about kSuspendHintNs pass.
constexpr uint32_t kSuspendHintNs = 20000;
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(kSuspendHintNs)
      : "memory");
  return ok != 0;
}
// Waits for the phase with the given parity to complete; gives up after about two
// seconds and returns false (the caller records kErrWaitTimeout and winds down).
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (clock64() - t0 > kWaitLimitCycles) return false;
  }
}

// ---------------------------------------------------------------- bulk copy (TMA, 1-D)
// Global -> shared copy of `bytes` (multiple of 16, both addresses 16-byte aligned),
// completion counted on `bar` in bytes.
__device__ __forceinline__ void bulk_g2s(void* dst_smem, const void* src_gmem, uint32_t bytes,
                                         uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst_smem)),
      "l"(src_gmem), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// The same copy with an L2 eviction-priority policy (from l2_evict_first_policy).
__device__ __forceinline__ void bulk_g2s_hint(void* dst_smem, const void* src_gmem, uint32_t bytes, uint64_t* bar,
                                              uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::"r"(
          smem_u32(dst_smem)),
      "l"(src_gmem), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}
// L2 policy for data read once per call (the state tiles): evict it first, so that it
// does not push the ring records and this call's inputs out of L2.
__device__ __forceinline__ uint64_t l2_evict_first_policy() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

// L2 policy for everything else the kernel reads (ring records, queries): normal priority.
__device__ __forceinline__ uint64_t l2_evict_normal_policy() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_normal.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

// ---------------------------------------------------------------- cp.async (LDGSTS)
// Small global -> shared copies issued per thread; their completion is tracked by an
// mbarrier through cp_async_arrive (each issuing thread arrives once per phase).
__device__ __forceinline__ void cp_async16(void* dst_smem, const void* src_gmem) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst_smem)), "l"(src_gmem) : "memory");
}
__device__ __forceinline__ void cp_async4(void* dst_smem, const void* src_gmem) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(dst_smem)), "l"(src_gmem) : "memory");
}
// Arrive on `bar` once this thread's earlier cp.async copies have landed (the barrier's
// expected arrival count includes this arrival).
__device__ __forceinline__ void cp_async_arrive(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// ---------------------------------------------------------------- consumer-group barriers
// Named barrier `id` (1 + group) spans the `count` threads of one consumer group only.
__device__ __forceinline__ void group_sync(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}
// Group barrier with an AND-vote across the group's threads.
__device__ __forceinline__ bool group_all(bool v, int id, int count) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)v), "r"(id), "r"(count)
      : "memory");
  return r != 0;
}

// ---------------------------------------------------------------- conversions
template <typename IO>
struct IoT;
template <>
struct IoT<float> {
  static constexpr int bytes = 4;
  __device__ __forceinline__ static float4 load4(const void* p) {
    return *reinterpret_cast<const float4*>(p);
  }
  __device__ __forceinline__ static float load1(const void* p) { return *reinterpret_cast<const float*>(p); }
  __device__ __forceinline__ static float2 load2(const void* p) { return *reinterpret_cast<const float2*>(p); }
};
template <>
struct IoT<__nv_bfloat16> {
  static constexpr int bytes = 2;
  __device__ __forceinline__ static float4 load4(const void* p) {
    const uint2 u = *reinterpret_cast<const uint2*>(p);
    const __nv_bfloat162 lo = *reinterpret_cast<const __nv_bfloat162*>(&u.x);
    const __nv_bfloat162 hi = *reinterpret_cast<const __nv_bfloat162*>(&u.y);
    const float2 a = __bfloat1622float2(lo);
    const float2 b = __bfloat1622float2(hi);
    return make_float4(a.x, a.y, b.x, b.y);
  }
  __device__ __forceinline__ static float load1(const void* p) {
    return __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(p));
  }
  __device__ __forceinline__ static float2 load2(const void* p) {
    return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(p));
  }
};

// four e4m3 codes (byte i = element i) -> four floats
__device__ __forceinline__ float4 e4m3x4_to_float4(uint32_t w) {
  const __half2_raw lo = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(w & 0xFFFFu), __NV_E4M3);
  const __half2_raw hi = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(w >> 16), __NV_E4M3);
  const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&lo));
  const float2 b = __half22float2(*reinterpret_cast<const __half2*>(&hi));
  return make_float4(a.x, a.y, b.x, b.y);
}
// one float -> e4m3 code, round to nearest even, saturating to +-448
__device__ __forceinline__ uint32_t float_to_e4m3(float x) {
  return static_cast<uint32_t>(__nv_cvt_float_to_fp8(x, __NV_SATFINITE, __NV_E4M3));
}
// quantise four values of one row with that row's inverse scale; byte i = element i
__device__ __forceinline__ uint32_t quant4_e4m3(float4 x, float inv) {
  return float_to_e4m3(__fmul_rn(x.x, inv)) | (float_to_e4m3(__fmul_rn(x.y, inv)) << 8) |
         (float_to_e4m3(__fmul_rn(x.z, inv)) << 16) | (float_to_e4m3(__fmul_rn(x.w, inv)) << 24);
}
// row scale and its inverse from the row's largest magnitude (1 and 1 for a zero row)
__device__ __forceinline__ void e4m3_row_scale(float amax, float& scale, float& inv) {
  if (amax > 0.f) {
    scale = __fdiv_rn(amax, 448.f);
    inv = __fdiv_rn(448.f, amax);
  } else {
    scale = 1.f;
    inv = 1.f;
  }
}

// FP4 e2m1 read copy: four codes in 16 bits, element 2i in the low nibble of byte i, 2i+1
// in its high nibble; the hardware conversions (cvt .e2m1x2) pack the first operand into
// the upper nibble and unpack the upper nibble into the upper half.
__device__ __forceinline__ float4 e2m1x4_to_float4(uint32_t w16) {
  uint32_t h01, h23;
  asm("{\n\t.reg .b8 lo, hi;\n\t"
      "mov.b16 {lo, hi}, %2;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, lo;\n\t"
      "cvt.rn.f16x2.e2m1x2 %1, hi;\n\t}"
      : "=r"(h01), "=r"(h23)
      : "h"(static_cast<unsigned short>(w16)));
  const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&h01));
  const float2 b = __half22float2(*reinterpret_cast<const __half2*>(&h23));
  return make_float4(a.x, a.y, b.x, b.y);
}
// four values of one row, times that row's inverse scale, to e2m1 codes (round to nearest
// even, saturating to +-6); returns 16 bits
__device__ __forceinline__ uint32_t quant4_e2m1(float4 x, float inv) {
  unsigned short out;
  asm("{\n\t.reg .b8 lo, hi;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 lo, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 hi, %4, %3;\n\t"
      "mov.b16 %0, {lo, hi};\n\t}"
      : "=h"(out)
      : "f"(__fmul_rn(x.x, inv)), "f"(__fmul_rn(x.y, inv)), "f"(__fmul_rn(x.z, inv)), "f"(__fmul_rn(x.w, inv)));
  return out;
}
// row scale and its inverse for the e2m1 copy (largest magnitude 6; 1 and 1 for a zero row)
__device__ __forceinline__ void e2m1_row_scale(float amax, float& scale, float& inv) {
  if (amax > 0.f) {
    scale = __fdiv_rn(amax, 6.f);
    inv = __fdiv_rn(6.f, amax);
  } else {
    scale = 1.f;
    inv = 1.f;
  }
}

__device__ __forceinline__ float dot4(float4 a, float4 b) {
  return fmaf(a.x, b.x, fmaf(a.y, b.y, fmaf(a.z, b.z, a.w * b.w)));
}
// Read-copy codes for the dot products: four e4m3 (byte i = element i) or e2m1 codes as
// two f16x2 words (elements 0,1 and 2,3), the first step of the conversions above
// without the widening to f32.
__device__ __forceinline__ uint2 e4m3x4_to_half4(uint32_t w) {
  const __half2_raw lo = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(w & 0xFFFFu), __NV_E4M3);
  const __half2_raw hi = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(w >> 16), __NV_E4M3);
  return make_uint2(*reinterpret_cast<const uint32_t*>(&lo), *reinterpret_cast<const uint32_t*>(&hi));
}
__device__ __forceinline__ uint2 e2m1x4_to_half4(uint32_t w16) {
  uint32_t h01, h23;
  asm("{\n\t.reg .b8 lo, hi;\n\t"
      "mov.b16 {lo, hi}, %2;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, lo;\n\t"
      "cvt.rn.f16x2.e2m1x2 %1, hi;\n\t}"
      : "=r"(h01), "=r"(h23)
      : "h"(static_cast<unsigned short>(w16)));
  return make_uint2(h01, h23);
}
// four floats (exactly representable in f16: BF16 inputs in f16's range) as two f16x2 words
__device__ __forceinline__ uint2 float4_to_half4(float4 v) {
  const __half2 lo = __floats2half2_rn(v.x, v.y);
  const __half2 hi = __floats2half2_rn(v.z, v.w);
  return make_uint2(*reinterpret_cast<const uint32_t*>(&lo), *reinterpret_cast<const uint32_t*>(&hi));
}
// a.x b.x + (a.y b.y + (a.z b.z + a.w b.w)) of f16 operands, accumulated in f32 by the
// mixed-precision FMA (f16 x f16 -> f32): every product is exact in f32, so the result
// equals dot4 of the operands widened to f32, without the widening conversions.
__device__ __forceinline__ float dot4_h(uint2 a, uint2 b) {
  float d;
  asm("{\n\t.reg .b16 a0, a1, a2, a3, b0, b1, b2, b3;\n\t"
      "mov.b32 {a0, a1}, %1;\n\t"
      "mov.b32 {a2, a3}, %2;\n\t"
      "mov.b32 {b0, b1}, %3;\n\t"
      "mov.b32 {b2, b3}, %4;\n\t"
      "fma.rn.f32.f16 %0, a3, b3, 0f00000000;\n\t"
      "fma.rn.f32.f16 %0, a2, b2, %0;\n\t"
      "fma.rn.f32.f16 %0, a1, b1, %0;\n\t"
      "fma.rn.f32.f16 %0, a0, b0, %0;\n\t}"
      : "=f"(d)
      : "r"(a.x), "r"(a.y), "r"(b.x), "r"(b.y));
  return d;
}
__device__ __forceinline__ float amax4(float4 a) {
  return fmaxf(fmaxf(fabsf(a.x), fabsf(a.y)), fmaxf(fabsf(a.z), fabsf(a.w)));
}

// ---------------------------------------------------------------- warp scans
// Inclusive suffix product over the lanes of a warp: lane l gets x_l * x_{l+1} * ... * x_31.
__device__ __forceinline__ float warp_suffix_prod(float x, int lane) {
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const float t = __shfl_down_sync(0xffffffffu, x, off);
    if (lane + off < 32) x *= t;
  }
  return x;
}

// ---------------------------------------------------------------- segment reductions
// Maximum over the TPR lanes of an aligned lane segment (all lanes get it).
template <int TPR>
__device__ __forceinline__ float seg_allmax(float v) {
#pragma unroll
  for (int off = TPR / 2; off >= 1; off >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, off));
  return v;
}

// Transposing reduction: each lane of a TPR-lane segment holds R partial sums (one per
// row it covers); afterwards lane l holds complete row sums for R/TPR rows (or one row,
// replicated over TPR/R lanes, when R < TPR). Costs about R + log2(TPR) shuffles
// instead of R * log2(TPR). `base` returns the index of the first row held in v[0].
// (MAX: the same with the maximum in place of the sum.)
template <int R, int OFF, bool MAX = false>
struct SegTranspose {
  __device__ __forceinline__ static float op(float a, float b) { return MAX ? fmaxf(a, b) : a + b; }
  __device__ __forceinline__ static void run(float* v, int lane, int& base) {
    if constexpr (OFF >= 1) {
      if constexpr (R > 1) {
        constexpr int H = R / 2;
        const bool up = (lane & OFF) != 0;
#pragma unroll
        for (int i = 0; i < H; ++i) {
          const float send = up ? v[i] : v[i + H];
          const float keep = up ? v[i + H] : v[i];
          v[i] = op(keep, __shfl_xor_sync(0xffffffffu, send, OFF));
        }
        if (up) base += H;
        SegTranspose<H, OFF / 2, MAX>::run(v, lane, base);
      } else {
        v[0] = op(v[0], __shfl_xor_sync(0xffffffffu, v[0], OFF));
        SegTranspose<1, OFF / 2, MAX>::run(v, lane, base);
      }
    }
  }
};
template <int R>
struct SegLog2 {
  static constexpr int value = (R <= 1) ? 0 : 1 + SegLog2<R / 2>::value;
};
template <>
struct SegLog2<1> {
  static constexpr int value = 0;
};

template <int R, int TPR, bool MAX = false>
struct SegReduce {
  static constexpr int kHeld = (R >= TPR) ? R / TPR : 1;  // row sums each lane ends with
  // returns true for the lanes that should write their v[0..kHeld)
  __device__ __forceinline__ static bool run(float* v, int lane, int& base) {
    base = 0;
    SegTranspose<R, TPR / 2, MAX>::run(v, lane, base);
    if constexpr (R >= TPR) {
      return true;
    } else {
      return (lane & (TPR / R - 1)) == 0;
    }
  }
};

}  // namespace replay
