// decode.cu -- the single-token recurrent step (decode): for every head,
//   P = S Diag(alpha),  e = v - P k,  S <- P + beta e k^T,  o = S q,
// the gated delta-rule update itself, applied to one token with the fp32
// state updated in place.  Each state row a (value index) is independent:
//   s_a <- s_a o alpha,  e_a = v_a - s_a . k,  s_a <- s_a + beta e_a k,  o_a = s_a . q,
// so a warp owns four rows (128 keys = 4 per lane: four 512-byte loads in
// flight, then two warp reductions per row).  The step is HBM-bound: it reads and
// writes the d_v x d_k fp32 state once per token.  In Kaczmarz mode
// beta = eta / (||k||^2 + eps), each warp forming ||k||^2 itself.  With the
// SFDA phase gate (PHASE) the decay is the 2 x 2 rotation-decay block of each
// key pair, (x, y) <- alpha (cos theta x - sin theta y, sin theta x + cos theta y)
// (the explainer's Lambda_t = diag(alpha e^{i theta}) in real coordinates); a
// lane's four keys are two whole pairs.

#include "dr_common.cuh"

namespace dr {
namespace {

constexpr int kDecodeThreads = 256;  // 8 warps per block
constexpr int kRows = 4;             // state rows per warp

template <typename T>
__device__ __forceinline__ float4 load4(const T* p);
template <>
__device__ __forceinline__ float4 load4<float>(const float* p) {
  return *reinterpret_cast<const float4*>(p);
}
template <>
__device__ __forceinline__ float4 load4<__nv_bfloat16>(const __nv_bfloat16* p) {
  const uint2 r = *reinterpret_cast<const uint2*>(p);
  const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&r.x));
  const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&r.y));
  return make_float4(a.x, a.y, b.x, b.y);
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

template <typename T, bool PHASE>
__global__ void __launch_bounds__(kDecodeThreads)
    k_decode_step(Problem p, const T* __restrict__ q, const T* __restrict__ k,
                  const T* __restrict__ v, const float* __restrict__ beta,
                  const float* __restrict__ g, float* __restrict__ S, T* __restrict__ o) {
  const int lane = threadIdx.x & 31;
  // kRows consecutive state rows per warp (dv is a multiple of 16, so they
  // share one head); all their loads are issued before any arithmetic
  const long row0 = ((long)blockIdx.x * (kDecodeThreads / 32) + (threadIdx.x >> 5)) * kRows;
  if (row0 >= (long)p.B * p.H * p.dv) return;
  const long head = row0 / p.dv;  // b * H + h (T = 1)
  const int a0 = (int)(row0 % p.dv);
  const int c0 = 4 * lane;
  const bool act = c0 < p.dk;
  float4 s[kRows];
  float4 kk = make_float4(0.f, 0.f, 0.f, 0.f), qq = kk;
  float4 al = make_float4(1.f, 1.f, 1.f, 1.f);
  float4 rot = make_float4(0.f, 0.f, 0.f, 0.f);  // PHASE: (a cos, a sin) of the two pairs
  float* srow = S + row0 * p.dk;
#pragma unroll
  for (int r = 0; r < kRows; ++r)
    s[r] = act ? __ldcs(reinterpret_cast<const float4*>(srow + r * p.dk + c0))
               : make_float4(0.f, 0.f, 0.f, 0.f);
  if (act) {
    kk = load4<T>(k + head * p.dk + c0);
    qq = load4<T>(q + head * p.dk + c0);
    if (PHASE) {
      const float4 gg = *reinterpret_cast<const float4*>(g + head * p.dk + c0);
      float s0, c0r, s1, c1r;
      sincosf(gg.y, &s0, &c0r);
      sincosf(gg.w, &s1, &c1r);
      const float a0 = __expf(gg.x), a1 = __expf(gg.z);
      rot = make_float4(a0 * c0r, a0 * s0, a1 * c1r, a1 * s1);
    } else if (p.gate == kGateChannel) {
      const float4 gg = *reinterpret_cast<const float4*>(g + head * p.dk + c0);
      al = make_float4(__expf(gg.x), __expf(gg.y), __expf(gg.z), __expf(gg.w));
    } else if (p.gate == kGateScalar) {
      const float e = __expf(g[head]);
      al = make_float4(e, e, e, e);
    }
  }
  float vr[kRows];
#pragma unroll
  for (int r = 0; r < kRows; ++r) vr[r] = load_f(v + head * p.dv + a0 + r);
  float b = beta[head];
  if (p.beta_mode == kBetaKaczmarz) {
    const float nn = warp_sum(kk.x * kk.x + kk.y * kk.y + kk.z * kk.z + kk.w * kk.w);
    b = b / (nn + p.eps);
  }
  float pk[kRows];
#pragma unroll
  for (int r = 0; r < kRows; ++r) {
    if (PHASE) {
      const float x0 = s[r].x, y0 = s[r].y, x1 = s[r].z, y1 = s[r].w;
      s[r].x = rot.x * x0 - rot.y * y0;
      s[r].y = rot.y * x0 + rot.x * y0;
      s[r].z = rot.z * x1 - rot.w * y1;
      s[r].w = rot.w * x1 + rot.z * y1;
    } else {
      s[r].x *= al.x;
      s[r].y *= al.y;
      s[r].z *= al.z;
      s[r].w *= al.w;
    }
    pk[r] = s[r].x * kk.x + s[r].y * kk.y + s[r].z * kk.z + s[r].w * kk.w;
  }
#pragma unroll
  for (int r = 0; r < kRows; ++r) pk[r] = warp_sum(pk[r]);
  float oa[kRows];
#pragma unroll
  for (int r = 0; r < kRows; ++r) {
    const float be = b * (vr[r] - pk[r]);
    s[r].x += be * kk.x;
    s[r].y += be * kk.y;
    s[r].z += be * kk.z;
    s[r].w += be * kk.w;
    oa[r] = s[r].x * qq.x + s[r].y * qq.y + s[r].z * qq.z + s[r].w * qq.w;
    if (act) __stcs(reinterpret_cast<float4*>(srow + r * p.dk + c0), s[r]);
  }
#pragma unroll
  for (int r = 0; r < kRows; ++r) oa[r] = warp_sum(oa[r]);
  if (lane < kRows) {
    float x = oa[0];
#pragma unroll
    for (int r = 1; r < kRows; ++r)
      if (lane == r) x = oa[r];
    store_f(o + head * p.dv + a0 + lane, x);
  }
}

}  // namespace

cudaError_t launch_decode_step(const Problem& p, int bf16, const void* q, const void* k,
                               const void* v, const float* beta, const float* g, float* S, void* o,
                               cudaStream_t st) {
  const long rows = (long)p.B * p.H * p.dv;
  const int rows_per_block = kDecodeThreads / 32 * kRows;
  const unsigned blocks = (unsigned)((rows + rows_per_block - 1) / rows_per_block);
  const double heads = (double)p.B * p.H, es = bf16 ? 2.0 : 4.0;
  // reads and writes the fp32 state; reads q, k, v, beta, g; writes o
  const double bytes = heads * (2.0 * p.dv * p.dk * 4 + (2.0 * p.dk + 2.0 * p.dv) * es + 4 +
                                (p.gate == kGateChannel || p.gate == kGatePhase ? p.dk * 4
                                 : p.gate == kGateScalar                        ? 4
                                                                                : 0));
  const double flops = heads * p.dv * p.dk * 7.0;
  prof_begin(kKDecode, bytes, bytes, flops, st);  // all of it is operator I/O
  using bf = __nv_bfloat16;
  if (p.gate == kGatePhase) {
    if (bf16)
      k_decode_step<bf, true><<<blocks, kDecodeThreads, 0, st>>>(
          p, (const bf*)q, (const bf*)k, (const bf*)v, beta, g, S, (bf*)o);
    else
      k_decode_step<float, true><<<blocks, kDecodeThreads, 0, st>>>(
          p, (const float*)q, (const float*)k, (const float*)v, beta, g, S, (float*)o);
  } else if (bf16) {
    k_decode_step<bf, false><<<blocks, kDecodeThreads, 0, st>>>(
        p, (const bf*)q, (const bf*)k, (const bf*)v, beta, g, S, (bf*)o);
  } else {
    k_decode_step<float, false><<<blocks, kDecodeThreads, 0, st>>>(
        p, (const float*)q, (const float*)k, (const float*)v, beta, g, S, (float*)o);
  }
  const cudaError_t e = cudaGetLastError();
  prof_end(st);
  return e;
}

}  // namespace dr
