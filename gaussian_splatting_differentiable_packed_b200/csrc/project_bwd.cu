// Projection backward ("Spirula Studio backward pass", section 5: each
// Gaussian's screen-space gradient goes back through the intrinsics and
// extrinsics to its six attributes: means, rotation, scale, opacity, DC and
// higher SH coefficients).
//
// One thread per Gaussian, 128 per CTA, looping over the cameras that see
// its Gaussian (the set bits of the packed projection's mask); a set bit
// gives the row by the same popcount arithmetic, so no (camera, Gaussian) ids
// are stored.  The gradient
// of the 3D covariance is summed over cameras first and taken through
// Sigma = M M^T, the scale and the quaternion once per Gaussian.
// Deterministic: no atomics.  Decisions that gate gradients (the Jacobian's
// off-axis clamp, the colour clamp) are re-taken with the forward's
// canonical arithmetic.
#include <cmath>

#include <cooperative_groups.h>

#include "ss_common.cuh"
#include "ss_math.cuh"

namespace ss {

constexpr int kCamChunkB = 32;

// dL/d(coefficient k, channel ch) += b_k v_ch where the channel was not
// clamped (vm holds v with the clamped channels zeroed).
template <int DEG>
__device__ __forceinline__ void sh_coef_grads(float X, float Y, float Z, const float vm[3], const bool cl[3],
                                              float* gsh) {
  constexpr int K = (DEG + 1) * (DEG + 1);
  float b[16];
  sh_basis(DEG, X, Y, Z, b);
#pragma unroll
  for (int k = 0; k < K; ++k)
#pragma unroll
    for (int ch = 0; ch < 3; ++ch)
      if (!cl[ch]) gsh[3 * k + ch] += b[k] * vm[ch];
}

// The view direction's gradient sum_k w_k db_k/d(X, Y, Z) with
// w_k = sum_ch coefficient(k, ch) v_ch (one weight per basis function; only
// the derivatives that are not identically zero are taken).
template <int DEG>
__device__ __forceinline__ void sh_dir_grads(float X, float Y, float Z, const float* __restrict__ shn,
                                             const float vm[3], float vdir[3]) {
  constexpr int K = (DEG + 1) * (DEG + 1);
  float w[16];
#pragma unroll
  for (int k = 0; k < K; ++k)
    w[k] = k == 0 ? 0.0f : shn[3 * k] * vm[0] + shn[3 * k + 1] * vm[1] + shn[3 * k + 2] * vm[2];
  float gX = 0.0f, gY = 0.0f, gZ = 0.0f;
  if (DEG >= 1) {
    gY -= SS_SH_C1 * w[1];
    gZ += SS_SH_C1 * w[2];
    gX -= SS_SH_C1 * w[3];
  }
  if (DEG >= 2) {
    gX += SS_SH_C2A * (Y * w[4] - Z * w[7]) + 2.0f * SS_SH_C2E * X * w[8] - 2.0f * SS_SH_C2C * X * w[6];
    gY += SS_SH_C2A * (X * w[4] - Z * w[5]) - 2.0f * SS_SH_C2E * Y * w[8] - 2.0f * SS_SH_C2C * Y * w[6];
    gZ += -SS_SH_C2A * (Y * w[5] + X * w[7]) + 4.0f * SS_SH_C2C * Z * w[6];
  }
  if (DEG >= 3) {
    const float XX = X * X, YY = Y * Y, ZZ = Z * Z;
    gX += -SS_SH_C3A * 6.0f * X * Y * w[9] + SS_SH_C3B * Y * Z * w[10] + 2.0f * SS_SH_C3C * X * Y * w[11] -
          6.0f * SS_SH_C3D * X * Z * w[12] - SS_SH_C3C * (4.0f * ZZ - 3.0f * XX - YY) * w[13] +
          2.0f * SS_SH_C3F * X * Z * w[14] - SS_SH_C3A * (3.0f * XX - 3.0f * YY) * w[15];
    gY += -SS_SH_C3A * (3.0f * XX - 3.0f * YY) * w[9] + SS_SH_C3B * X * Z * w[10] -
          SS_SH_C3C * (4.0f * ZZ - XX - 3.0f * YY) * w[11] - 6.0f * SS_SH_C3D * Y * Z * w[12] +
          2.0f * SS_SH_C3C * X * Y * w[13] - 2.0f * SS_SH_C3F * Y * Z * w[14] + SS_SH_C3A * 6.0f * X * Y * w[15];
    gZ += SS_SH_C3B * X * Y * w[10] - 8.0f * SS_SH_C3C * Y * Z * w[11] +
          SS_SH_C3D * (6.0f * ZZ - 3.0f * XX - 3.0f * YY) * w[12] - 8.0f * SS_SH_C3C * X * Z * w[13] +
          SS_SH_C3F * (XX - YY) * w[14];
  }
  vdir[0] = gX;
  vdir[1] = gY;
  vdir[2] = gZ;
}

// Shared-memory stride per Gaussian for SH blocks (odd, so that thread t's
// word k sits in bank (t*stride + k) mod 32: conflict-free across a warp).
template <int DEG>
__host__ __device__ constexpr int sh_stride() {
  return ((3 * (DEG + 1) * (DEG + 1)) % 2 == 0) ? 3 * (DEG + 1) * (DEG + 1) + 1 : 3 * (DEG + 1) * (DEG + 1);
}

// Gaussian gi and coefficient q of word u (0..3) of the SH block's 16-byte
// vector v (word f = 4v + u: gi = f / K3, q = f mod K3).  When K3 is a
// multiple of 4 no vector straddles two Gaussians, so the division is taken
// once per vector rather than once per word.
template <int K3>
__device__ __forceinline__ void sh_word(int v, int u, int& gi, int& q) {
  if constexpr (K3 % 4 == 0) {
    gi = v / (K3 / 4);
    q = 4 * (v - gi * (K3 / 4)) + u;
  } else {
    const int f = 4 * v + u;
    gi = f / K3;
    q = f - gi * K3;
  }
}

// Fused optimizer step (the pages' "fused projection backward + optimizer":
// the gradient sums never leave registers / shared memory).  Adam with bias
// correction on the raw parameters: means, quaternions, log-scales,
// logit-opacities and SH coefficients; the kernel also refreshes the activated
// copies (scales = exp, opacities = sigmoid) that the next forward reads.
struct AdamArgs {
  float *m_means, *v_means, *m_quats, *v_quats, *m_scales, *v_scales, *m_opac, *v_opac, *m_sh, *v_sh;
  float *means, *quats, *log_scales, *scales, *logit_opac, *opac, *sh;  // updated in place
  float lr_means, lr_quats, lr_scales, lr_opac, lr_sh_dc, lr_sh_rest;
  float b1, b2, eps;
  float ibc1;   // 1 / (1 - beta1^t)
  float ibc2s;  // 1 / sqrt(1 - beta2^t)
};

// One Adam update of parameter p with gradient g; m and v are updated in place.
// The square root and the quotient come from the hardware's approximate
// reciprocal square root and divide (a few ulp on the step, far inside the
// update's tolerance; v >= 0, and v = 0 gives the root 0).
__device__ __forceinline__ float adam_update(float p, float g, float& m, float& v, float lr, const AdamArgs& a) {
  m = a.b1 * m + (1.0f - a.b1) * g;
  v = a.b2 * v + (1.0f - a.b2) * g * g;
  const float root = v > 0.0f ? v * rsqrtf(v) : 0.0f;
  return p - __fdividef(lr * (m * a.ibc1), root * a.ibc2s + a.eps);
}

// Block-quantised gradient accumulation ("Spirula Studio backward pass",
// section 6, technique 1: each attribute's accumulator is kept as 16-bit
// codes in blocks of 256 Gaussians, and every sub-batch's projection
// backward decodes it, adds the sub-batch's gradient and quantises again, so
// no fp32 gradient array exists).  One scale per (attribute, block) = the
// block's largest magnitude / 32767 and codes = nearest-even(x / scale); an
// all-zero block has scale 0.  A block of 256 Gaussians is two CTAs, launched
// as a cluster of two that exchange their maxima through distributed shared
// memory.  Attributes: means [N][3], quats [N][4], scales [N][3], opacities
// [N], SH DC [N][3], higher SH [N][K-1][3].
constexpr int kGqAttr = 6;
constexpr int64_t kGqBlock = 256;
constexpr float kGqMax = 32767.0f;

struct GqArgs {
  int16_t* code[kGqAttr];
  float* scale;  // [kGqAttr][ceil(N / 256)]
  int first;     // the accumulators start from zero (their contents are ignored)
};

// Code of x at a block scale s, given is = 1/s (0 when s is 0): the quotient
// x/s is taken as x * is, at most about 1.5 ulp of the quotient (0.005 of a
// step at full scale) from the correctly rounded one.
__device__ __forceinline__ int16_t gq_code(float x, float is) {
  return (int16_t)__float2int_rn(fminf(fmaxf(x * is, -kGqMax), kGqMax));
}

// Largest value of v over the CTA for each attribute (a < kGqAttr), into out.
__device__ __forceinline__ void gq_cta_max(const float (&v)[kGqAttr], float (*wmax)[kBlock / 32], float* out) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int a = 0; a < kGqAttr; ++a) {
    float m = v[a];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (lane == 0) wmax[a][warp] = m;
  }
  __syncthreads();
  if (threadIdx.x < kGqAttr) {
    float m = 0.0f;
#pragma unroll
    for (int w = 0; w < kBlock / 32; ++w) m = fmaxf(m, wmax[threadIdx.x][w]);
    out[threadIdx.x] = m;
  }
}

// The pair's maxima: both CTAs of the cluster have written theirs to amax;
// every thread reads the partner's and returns the block's scales.  The
// second cluster barrier keeps a CTA's maxima alive until its partner has
// read them.  Every thread of both CTAs calls this exactly once.
__device__ __forceinline__ void gq_exchange(float* amax, float (&scale)[kGqAttr]) {
  namespace cg = cooperative_groups;
  cg::cluster_group cl = cg::this_cluster();
  cl.sync();
  const float* other = cl.map_shared_rank(amax, (int)(cl.block_rank() ^ 1u));
#pragma unroll
  for (int a = 0; a < kGqAttr; ++a) scale[a] = fmaxf(amax[a], other[a]) / kGqMax;
  cl.sync();
}

template <int DEG, bool ADAM, bool GQ>
__global__ __launch_bounds__(kBlock, 4) void k_project_bwd(Geo g, const float* __restrict__ cams,
                                                           const float* __restrict__ means,
                                                           const float* __restrict__ quats,
                                                           const float* __restrict__ scales,
                                                           const float* __restrict__ sh,
                                                           const uint32_t* __restrict__ mask,
                                                           const int64_t* __restrict__ block_off,
                                                           const float* __restrict__ v_screen,
                                                           float* __restrict__ v_means, float* __restrict__ v_quats,
                                                           float* __restrict__ v_scales, float* __restrict__ v_opac,
                                                           float* __restrict__ v_sh, const float* __restrict__ opacities,
                                                           AdamArgs adam, int64_t ahead, GqArgs gqa) {
  constexpr int K = (DEG + 1) * (DEG + 1);
  constexpr int K3 = 3 * K;
  constexpr int KP = sh_stride<DEG>();
  constexpr int kWarps = kBlock / 32;
  __shared__ float s_gq_wmax[GQ ? kGqAttr : 1][kWarps];
  __shared__ float s_gq_amax[GQ ? kGqAttr : 1];
  __shared__ Cam scam[kCamChunkB];
  __shared__ uint32_t s_word[kCamChunkB][kWarps];
  __shared__ int64_t s_row0[kCamChunkB][kWarps];
  __shared__ float s_margin[kBlock][3];
  // the optimizer updates every parameter and the accumulators are decoded
  // into the SH staging area, so only the plain backward skips unseen rows
  constexpr bool kSkipUnseen = !ADAM && !GQ;
  extern __shared__ float smem[];
  float* sh_s = smem;                 // [kBlock][KP] SH coefficients of the CTA's Gaussians
  float* gsh_s = smem + kBlock * KP;  // [kBlock][KP] their gradient accumulators
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t blk = blockIdx.x;
  const int64_t n0 = blk * kBlock;
  const int64_t n = n0 + threadIdx.x;
  const bool valid = n < g.N;
  const int cnt = (int)min64(kBlock, g.N - n0);
  if constexpr (GQ) {
    if (blk >= g.blocks_per_cam) {
      // the cluster's second CTA past the last block of Gaussians (an odd
      // block count): no Gaussians, but it takes part in the pair's exchange
      if (threadIdx.x < kGqAttr) s_gq_amax[threadIdx.x] = 0.0f;
      float scale[kGqAttr];
      gq_exchange(s_gq_amax, scale);
      return;
    }
  }
  // the CTA's gradient rows of camera c are the contiguous rows
  // block_off[c][blk] .. block_off[c][blk + 1]: have L2 fetch them now, the
  // camera loop reads them one pair at a time
  for (int c = threadIdx.x; c < g.C; c += kBlock) {
    const int64_t r0 = block_off[(int64_t)c * g.blocks_per_cam + blk];
    const int64_t r1 = block_off[(int64_t)c * g.blocks_per_cam + blk + 1];
    prefetch_l2(v_screen + r0 * kRowF, (uint32_t)((r1 - r0) * kRowF * 4));
  }
  // (blocks_per_cam, not the grid: a grad-quant grid may hold one CTA more)
  const bool prefetch_ahead = ahead > 0 && blk + ahead < (GQ ? g.blocks_per_cam : (int64_t)gridDim.x);
  if (prefetch_ahead && threadIdx.x == 0) {
    // the SH block of the CTA that starts about a wave later, into L2
    const int64_t m0 = (blk + ahead) * kBlock;
    prefetch_l2(sh + m0 * K3, (uint32_t)(min64(kBlock, g.N - m0) * K3 * 4));
  }
  // The camera chunk of the first cameras: each warp's mask word and first
  // row per camera (loaded before the SH block, so the plain backward knows
  // which Gaussians some camera sees; later chunks are loaded in the loop).
  // Every warp loads its own words and first rows (lane cc: camera c0 + cc,
  // the CTA's four mask words of that camera in one 16-byte load, so a
  // warp's rows need no chain of loads); warp 0 also loads the cameras.
  static_assert(kWarps == 4, "one 16-byte load holds a CTA's mask words of a camera");
  auto load_chunk = [&](int c0) {
    const int nc = min(kCamChunkB, g.C - c0);
    if (threadIdx.x < nc) scam[threadIdx.x] = load_cam(cams + 20 * (int64_t)(c0 + threadIdx.x), g.W, g.H);
    if (lane < nc) {
      const int64_t c = c0 + lane;
      const uint4 wv = reinterpret_cast<const uint4*>(mask)[(c * g.n_pad + blk * kBlock) / 128];
      const int64_t row = block_off[c * g.blocks_per_cam + blk] + (warp > 0 ? __popc(wv.x) : 0) +
                          (warp > 1 ? __popc(wv.y) : 0) + (warp > 2 ? __popc(wv.z) : 0);
      s_word[lane][warp] = warp == 0 ? wv.x : warp == 1 ? wv.y : warp == 2 ? wv.z : wv.w;
      s_row0[lane][warp] = row;
    }
  };
  load_chunk(0);
  __syncthreads();  // the first chunk's words and rows are read by every warp
  // which of the warp's Gaussians any camera sees: with every camera in the
  // first chunk, from the words just staged; otherwise every row is read
  uint32_t seen_w = 0xFFFFFFFFu;
  if (kSkipUnseen && g.C <= kCamChunkB) seen_w = __reduce_or_sync(0xffffffffu, lane < g.C ? s_word[lane][warp] : 0u);
  if (GQ && !gqa.first && threadIdx.x == 0) {
    // the accumulator codes are read after the camera loop: have L2 fetch
    // the CTA's now
    constexpr int kWidths[kGqAttr] = {3, 4, 3, 1, 3, K3 - 3};
#pragma unroll
    for (int a = 0; a < kGqAttr; ++a)
      if (kWidths[a] > 0) prefetch_l2(gqa.code[a] + kWidths[a] * n0, (uint32_t)(cnt * kWidths[a] * 2));
  }
  if (ADAM && threadIdx.x == 0) {
    // the optimizer state is only touched after the camera loop: have L2 fetch
    // the CTA's moment blocks now, so the update reads them from L2
    prefetch_l2(adam.m_sh + n0 * K3, (uint32_t)(cnt * K3 * 4));
    prefetch_l2(adam.v_sh + n0 * K3, (uint32_t)(cnt * K3 * 4));
    prefetch_l2(adam.m_means + 3 * n0, (uint32_t)(cnt * 12));
    prefetch_l2(adam.v_means + 3 * n0, (uint32_t)(cnt * 12));
    prefetch_l2(adam.m_quats + 4 * n0, (uint32_t)(cnt * 16));
    prefetch_l2(adam.v_quats + 4 * n0, (uint32_t)(cnt * 16));
    prefetch_l2(adam.m_scales + 3 * n0, (uint32_t)(cnt * 12));
    prefetch_l2(adam.v_scales + 3 * n0, (uint32_t)(cnt * 12));
    prefetch_l2(adam.log_scales + 3 * n0, (uint32_t)(cnt * 12));
  }
  // staging of the warp's 32 rows of the CTA's SH block (contiguous and
  // 16-byte aligned: 32 * K3 floats a warp) with all 16-byte loads in flight
  // at once, a ragged warp word by word.  The plain backward skips the rows
  // of Gaussians no camera sees: their gradients are zero and their
  // coefficients are never read (a third of the Gaussians of the 15M-Gaussian
  // workload).  Each warp stages, walks and writes back its own rows, so no
  // CTA barrier separates them.
  const int wrows = max(0, min(32, cnt - 32 * warp));  // the warp's valid rows
  float* const sh_w = sh_s + 32 * warp * KP;
  float* const gsh_w = gsh_s + 32 * warp * KP;
  {
    const float* src = sh + (n0 + 32 * warp) * K3;
    if (wrows == 32) {
      constexpr int kV = 32 * K3 / 4;
      constexpr int kPer = (kV + 31) / 32;
      float4 buf[kPer];
#pragma unroll
      for (int r = 0; r < kPer; ++r) {
        const int v = lane + 32 * r;
        const bool need = v < kV && (!kSkipUnseen || ((seen_w >> ((4 * v) / K3)) & 1u) ||
                                     ((seen_w >> ((4 * v + 3) / K3)) & 1u));
        buf[r] = need ? reinterpret_cast<const float4*>(src)[v] : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int r = 0; r < kPer; ++r) {
        const int v = lane + 32 * r;
        if (v < kV) {
          const float e[4] = {buf[r].x, buf[r].y, buf[r].z, buf[r].w};
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            int gi, q;
            sh_word<K3>(v, u, gi, q);
            sh_w[gi * KP + q] = e[u];
            gsh_w[gi * KP + q] = 0.0f;
          }
        }
      }
    } else {
      for (int f = lane; f < 32 * K3; f += 32) {
        const int gi = f / K3, q = f - gi * K3;
        sh_w[gi * KP + q] = gi < wrows && (!kSkipUnseen || ((seen_w >> gi) & 1u)) ? src[f] : 0.0f;
        gsh_w[gi * KP + q] = 0.0f;
      }
    }
  }
  __syncwarp();  // the warp's staged rows are read by its lanes below
  {
    // Bound on how far 0.5 + sum_k sh_k b_k can move with the summation
    // order: each order's rounding is below 17 * 2^-24 * (0.5 + sum_k |sh_k
    // b_k|) and |b_k| <= 2 on the unit sphere for degree <= 3; the margin is
    // ten times that.  One per Gaussian and channel, read by the lane that
    // takes the pair.
    const float* shn = sh_s + threadIdx.x * KP;
#pragma unroll
    for (int ch = 0; ch < 3; ++ch) {
      float a = 0.0f;
#pragma unroll
      for (int kk = 0; kk < K; ++kk) a += fabsf(shn[3 * kk + ch]);
      s_margin[threadIdx.x][ch] = 1e-5f * (1.0f + 2.0f * a);
    }
  }
  const int64_t nn = valid ? n : 0;
  const float mx = means[3 * nn], my = means[3 * nn + 1], mz = means[3 * nn + 2];
  Cov3 S;
  {
    const float4 q = reinterpret_cast<const float4*>(quats)[nn];
    const QuatRot qr = quat_rot(q.x, q.y, q.z, q.w);
    S = cov3(qr, scales[3 * nn], scales[3 * nn + 1], scales[3 * nn + 2]);
  }
  float gmu[3] = {0.f, 0.f, 0.f}, go = 0.f;
  double gS[6] = {0., 0., 0., 0., 0., 0.};  // dL/dSigma, full-matrix convention (00 01 02 11 12 22)
  float gx[GQ ? 11 : 1] = {};  // GQ: this Gaussian's means, quats, scales and opacity gradients
  for (int c0 = 0; c0 < g.C; c0 += kCamChunkB) {
    const int nc = min(kCamChunkB, g.C - c0);
    if (c0 > 0) {  // the first chunk was loaded (and the CTA synchronised) before the SH block
      __syncthreads();
      load_chunk(c0);
      __syncthreads();
    }
    if (!valid) continue;
    // each lane walks the cameras of the chunk that see its Gaussian, in
    // camera order, with the next pair's gradient row loaded one pair ahead
    uint32_t vis = 0;
    for (int cc = 0; cc < nc; ++cc) vis |= ((s_word[cc][warp] >> lane) & 1u) << cc;
    const uint32_t below = (1u << lane) - 1u;
    const float* shn = sh_s + threadIdx.x * KP;
    float4 n0 = make_float4(0.f, 0.f, 0.f, 0.f), n1 = n0;
    float2 n2 = make_float2(0.f, 0.f);
    if (vis) {
      const int cc = __ffs(vis) - 1;
      const float* rp = v_screen + (s_row0[cc][warp] + __popc(s_word[cc][warp] & below)) * kRowF;
      n0 = reinterpret_cast<const float4*>(rp)[0];
      n1 = reinterpret_cast<const float4*>(rp)[1];
      n2 = reinterpret_cast<const float2*>(rp)[4];
    }
    while (vis) {
      const int cc = __ffs(vis) - 1;
      vis &= vis - 1;
      const float4 v0 = n0, v1 = n1;
      const float2 v2 = n2;
      if (vis) {
        const int cn = __ffs(vis) - 1;
        const float* rp = v_screen + (s_row0[cn][warp] + __popc(s_word[cn][warp] & below)) * kRowF;
        n0 = reinterpret_cast<const float4*>(rp)[0];
        n1 = reinterpret_cast<const float4*>(rp)[1];
        n2 = reinterpret_cast<const float2*>(rp)[4];
      }
      const Cam& k = scam[cc];
      const float* R = k.R;
      float px, py, pz;
      cam_point(k, mx, my, mz, px, py, pz);
      const float izc = rcp_(pz);
      const float u = mul(px, izc), v = mul(py, izc);
      const bool clx = (u < -k.limx) || (u > k.limx);
      const bool cly = (v < -k.limy) || (v > k.limy);
      const float ux = fminf(fmaxf(u, -k.limx), k.limx), uy = fminf(fmaxf(v, -k.limy), k.limy);
      const float iz = 1.0f / pz, iz2 = iz * iz;
      const float j00 = k.fx * iz, j02 = -j00 * ux, j11 = k.fy * iz, j12 = -j11 * uy;
      float T[6];
#pragma unroll
      for (int m = 0; m < 3; ++m) {
        T[m] = j00 * R[m] + j02 * R[6 + m];
        T[3 + m] = j11 * R[3 + m] + j12 * R[6 + m];
      }
      const double Sm[3][3] = {{S.s00, S.s01, S.s02}, {S.s01, S.s11, S.s12}, {S.s02, S.s12, S.s22}};
      double Td[6];
#pragma unroll
      for (int m = 0; m < 6; ++m) Td[m] = T[m];
      double TS[2][3];
#pragma unroll
      for (int r = 0; r < 2; ++r)
#pragma unroll
        for (int m = 0; m < 3; ++m)
          TS[r][m] = Td[3 * r] * Sm[0][m] + Td[3 * r + 1] * Sm[1][m] + Td[3 * r + 2] * Sm[2][m];
      const double a = TS[0][0] * Td[0] + TS[0][1] * Td[1] + TS[0][2] * Td[2] + 0.3;
      const double b = TS[0][0] * Td[3] + TS[0][1] * Td[4] + TS[0][2] * Td[5];
      const double cq = TS[1][0] * Td[3] + TS[1][1] * Td[4] + TS[1][2] * Td[5] + 0.3;
      const double id = 1.0 / (a * cq - b * b), id2 = id * id;
      const double vca = v0.z, vcb = v0.w, vcc = v1.x;
      const double va = (-vca * cq * cq + vcb * b * cq - vcc * b * b) * id2;
      const double vb = (2.0 * vca * b * cq - vcb * (a * cq + b * b) + 2.0 * vcc * a * b) * id2;
      const double vc = (-vca * b * b + vcb * a * b - vcc * a * a) * id2;
      const double hb = 0.5 * vb;
      float GT[2][3];
      double VT[2][3];
#pragma unroll
      for (int m = 0; m < 3; ++m) {
        GT[0][m] = (float)(2.0 * (va * TS[0][m] + hb * TS[1][m]));
        GT[1][m] = (float)(2.0 * (hb * TS[0][m] + vc * TS[1][m]));
        VT[0][m] = va * Td[m] + hb * Td[3 + m];
        VT[1][m] = hb * Td[m] + vc * Td[3 + m];
      }
      gS[0] += Td[0] * VT[0][0] + Td[3] * VT[1][0];
      gS[1] += Td[0] * VT[0][1] + Td[3] * VT[1][1];
      gS[2] += Td[0] * VT[0][2] + Td[3] * VT[1][2];
      gS[3] += Td[1] * VT[0][1] + Td[4] * VT[1][1];
      gS[4] += Td[1] * VT[0][2] + Td[4] * VT[1][2];
      gS[5] += Td[2] * VT[0][2] + Td[5] * VT[1][2];
      const float gj00 = GT[0][0] * R[0] + GT[0][1] * R[1] + GT[0][2] * R[2];
      const float gj02 = GT[0][0] * R[6] + GT[0][1] * R[7] + GT[0][2] * R[8];
      const float gj11 = GT[1][0] * R[3] + GT[1][1] * R[4] + GT[1][2] * R[5];
      const float gj12 = GT[1][0] * R[6] + GT[1][1] * R[7] + GT[1][2] * R[8];
      float gx_ = 0.f, gy = 0.f;
      float gz = -k.fx * iz2 * gj00 + k.fx * ux * iz2 * gj02 - k.fy * iz2 * gj11 + k.fy * uy * iz2 * gj12;
      const float gux = -k.fx * iz * gj02, guy = -k.fy * iz * gj12;
      if (!clx) { gx_ += gux * iz; gz -= gux * px * iz2; }
      if (!cly) { gy += guy * iz; gz -= guy * py * iz2; }
      const float vmx = v0.x, vmy = v0.y;
      gx_ += vmx * k.fx * iz; gz -= vmx * k.fx * px * iz2;
      gy += vmy * k.fy * iz; gz -= vmy * k.fy * py * iz2;
      gz += v2.y;
      gmu[0] += R[0] * gx_ + R[3] * gy + R[6] * gz;
      gmu[1] += R[1] * gx_ + R[4] * gy + R[7] * gz;
      gmu[2] += R[2] * gx_ + R[5] * gy + R[8] * gz;
      go += v1.y;
      float X = 0.f, Y = 0.f, Z = 0.f, il = 0.f;
      if (DEG > 0) view_dir(k, mx, my, mz, X, Y, Z, il);
      bool cl[3];
      {
        float bb[16];
        sh_basis(DEG, X, Y, Z, bb);
#pragma unroll
        for (int ch = 0; ch < 3; ++ch) {
          float f = 0.5f;
#pragma unroll
          for (int kk = 0; kk < K; ++kk) f = fmaf(shn[3 * kk + ch], bb[kk], f);
          bool c = !(f >= 0.0f);
          if (fabsf(f) <= s_margin[threadIdx.x][ch]) {
            float acc = mul(shn[ch], bb[0]);
#pragma unroll
            for (int kk = 1; kk < K; ++kk) acc = add(acc, mul(shn[3 * kk + ch], bb[kk]));
            c = !(add(acc, 0.5f) >= 0.0f);
          }
          cl[ch] = c;
        }
      }
      const float vr[3] = {v1.z, v1.w, v2.x};
      float vm[3];
#pragma unroll
      for (int ch = 0; ch < 3; ++ch) vm[ch] = cl[ch] ? 0.0f : vr[ch];
      sh_coef_grads<DEG>(X, Y, Z, vm, cl, gsh_s + threadIdx.x * KP);
      if (DEG > 0) {
        float vdir[3];
        sh_dir_grads<DEG>(X, Y, Z, shn, vm, vdir);
        const float dd = X * vdir[0] + Y * vdir[1] + Z * vdir[2];
        gmu[0] += (vdir[0] - X * dd) * il;
        gmu[1] += (vdir[1] - Y * dd) * il;
        gmu[2] += (vdir[2] - Z * dd) * il;
      }
    }
  }
  if (valid) {
    // the rotation and scales again (read back rather than kept live across
    // the camera walk)
    const float4 q4 = reinterpret_cast<const float4*>(quats)[n];
    const float s0 = scales[3 * n], s1 = scales[3 * n + 1], s2 = scales[3 * n + 2];
    const QuatRot qr = quat_rot(q4.x, q4.y, q4.z, q4.w);
    // Sigma = M M^T: dL/dM = 2 gS M, M = R_q diag(s)  (fp64, see above)
    const double Gs[3][3] = {{gS[0], gS[1], gS[2]}, {gS[1], gS[3], gS[4]}, {gS[2], gS[4], gS[5]}};
    const double sv[3] = {s0, s1, s2};
    double M[9];
#pragma unroll
    for (int i = 0; i < 3; ++i)
#pragma unroll
      for (int jj = 0; jj < 3; ++jj) M[3 * i + jj] = (double)qr.R[3 * i + jj] * sv[jj];
    double gsc[3] = {0., 0., 0.}, GR[9];
#pragma unroll
    for (int i = 0; i < 3; ++i)
#pragma unroll
      for (int jj = 0; jj < 3; ++jj) {
        const double gm = 2.0 * (Gs[i][0] * M[jj] + Gs[i][1] * M[3 + jj] + Gs[i][2] * M[6 + jj]);
        gsc[jj] += gm * qr.R[3 * i + jj];
        GR[3 * i + jj] = gm * sv[jj];
      }
    const double w = qr.w, x = qr.x, y = qr.y, z = qr.z;
    double vw = 0., vx = 0., vy = 0., vz = 0.;
    vy += -4.f * y * GR[0]; vz += -4.f * z * GR[0];
    vw += -2.f * z * GR[1]; vx += 2.f * y * GR[1]; vy += 2.f * x * GR[1]; vz += -2.f * w * GR[1];
    vw += 2.f * y * GR[2]; vx += 2.f * z * GR[2]; vy += 2.f * w * GR[2]; vz += 2.f * x * GR[2];
    vw += 2.f * z * GR[3]; vx += 2.f * y * GR[3]; vy += 2.f * x * GR[3]; vz += 2.f * w * GR[3];
    vx += -4.f * x * GR[4]; vz += -4.f * z * GR[4];
    vw += -2.f * x * GR[5]; vx += -2.f * w * GR[5]; vy += 2.f * z * GR[5]; vz += 2.f * y * GR[5];
    vw += -2.f * y * GR[6]; vx += 2.f * z * GR[6]; vy += -2.f * w * GR[6]; vz += 2.f * x * GR[6];
    vw += 2.f * x * GR[7]; vx += 2.f * w * GR[7]; vy += 2.f * z * GR[7]; vz += 2.f * y * GR[7];
    vx += -4.f * x * GR[8]; vy += -4.f * y * GR[8];
    const double dq = w * vw + x * vx + y * vy + z * vz;
    const double qi = qr.inv;
    const float gq[4] = {(float)((vw - w * dq) * qi), (float)((vx - x * dq) * qi), (float)((vy - y * dq) * qi),
                         (float)((vz - z * dq) * qi)};
    if constexpr (GQ) {
      gx[0] = gmu[0];
      gx[1] = gmu[1];
      gx[2] = gmu[2];
#pragma unroll
      for (int i = 0; i < 4; ++i) gx[3 + i] = gq[i];
#pragma unroll
      for (int i = 0; i < 3; ++i) gx[7 + i] = (float)gsc[i];
      gx[10] = go;
    } else if (!ADAM) {
      v_means[3 * n] = gmu[0];
      v_means[3 * n + 1] = gmu[1];
      v_means[3 * n + 2] = gmu[2];
      reinterpret_cast<float4*>(v_quats)[n] = make_float4(gq[0], gq[1], gq[2], gq[3]);
      v_scales[3 * n] = (float)gsc[0];
      v_scales[3 * n + 1] = (float)gsc[1];
      v_scales[3 * n + 2] = (float)gsc[2];
      v_opac[n] = go;
    } else {
      // means and raw quaternions take their gradients directly; log-scales
      // and logit-opacities through the activations (ds/dlog s = s,
      // do/dlogit = o (1 - o))
      const float mu[3] = {mx, my, mz};
#pragma unroll
      for (int i = 0; i < 3; ++i) {
        float m = adam.m_means[3 * n + i], v = adam.v_means[3 * n + i];
        adam.means[3 * n + i] = adam_update(mu[i], gmu[i], m, v, adam.lr_means, adam);
        adam.m_means[3 * n + i] = m;
        adam.v_means[3 * n + i] = v;
      }
      const float qv[4] = {q4.x, q4.y, q4.z, q4.w};
      float qn[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        float m = adam.m_quats[4 * n + i], v = adam.v_quats[4 * n + i];
        qn[i] = adam_update(qv[i], gq[i], m, v, adam.lr_quats, adam);
        adam.m_quats[4 * n + i] = m;
        adam.v_quats[4 * n + i] = v;
      }
      reinterpret_cast<float4*>(adam.quats)[n] = make_float4(qn[0], qn[1], qn[2], qn[3]);
      const float sc[3] = {s0, s1, s2};
#pragma unroll
      for (int i = 0; i < 3; ++i) {
        float m = adam.m_scales[3 * n + i], v = adam.v_scales[3 * n + i];
        const float ls = adam_update(adam.log_scales[3 * n + i], (float)gsc[i] * sc[i], m, v, adam.lr_scales, adam);
        adam.log_scales[3 * n + i] = ls;
        adam.scales[3 * n + i] = expf(ls);
        adam.m_scales[3 * n + i] = m;
        adam.v_scales[3 * n + i] = v;
      }
      const float o = opacities[n];
      float m = adam.m_opac[n], v = adam.v_opac[n];
      const float lo = adam_update(adam.logit_opac[n], go * o * (1.0f - o), m, v, adam.lr_opac, adam);
      adam.logit_opac[n] = lo;
      adam.opac[n] = 1.0f / (1.0f + expf(-lo));
      adam.m_opac[n] = m;
      adam.v_opac[n] = v;
    }
  }
  if (ADAM || GQ) __syncthreads();  // their epilogues run over the CTA's whole block
  if (ADAM) {
    // the CTA's SH block: Adam on each coefficient (DC with its own rate),
    // the staged values are the parameters.  A full block moves the moments
    // and parameters in 16-byte vectors, kChunk of them in flight per thread
    // (the block starts 16-byte aligned); the ragged last block word by word.
    const int64_t b0 = n0 * K3;
    if (cnt == kBlock) {
      constexpr int kV = kBlock * K3 / 4;
      constexpr int kChunk = (kV + kBlock - 1) / kBlock;  // every vector of the thread in flight
      float4* m4 = reinterpret_cast<float4*>(adam.m_sh + b0);
      float4* v4 = reinterpret_cast<float4*>(adam.v_sh + b0);
      float4* p4 = reinterpret_cast<float4*>(adam.sh + b0);
      for (int v0 = threadIdx.x; v0 < kV; v0 += kChunk * kBlock) {
        float4 mb[kChunk], vb[kChunk];
#pragma unroll
        for (int r = 0; r < kChunk; ++r) {
          const int vv = v0 + r * kBlock;
          if (vv < kV) {
            mb[r] = __ldcs(m4 + vv);
            vb[r] = __ldcs(v4 + vv);
          }
        }
#pragma unroll
        for (int r = 0; r < kChunk; ++r) {
          const int vv = v0 + r * kBlock;
          if (vv >= kV) continue;
          float me[4] = {mb[r].x, mb[r].y, mb[r].z, mb[r].w}, ve[4] = {vb[r].x, vb[r].y, vb[r].z, vb[r].w}, pe[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            int gi, q;
            sh_word<K3>(vv, u, gi, q);
            pe[u] = adam_update(sh_s[gi * KP + q], gsh_s[gi * KP + q], me[u], ve[u],
                                q < 3 ? adam.lr_sh_dc : adam.lr_sh_rest, adam);
          }
          // streaming stores: the lines are not read again in this kernel
          __stcs(p4 + vv, make_float4(pe[0], pe[1], pe[2], pe[3]));
          __stcs(m4 + vv, make_float4(me[0], me[1], me[2], me[3]));
          __stcs(v4 + vv, make_float4(ve[0], ve[1], ve[2], ve[3]));
        }
      }
    } else {
      for (int f = threadIdx.x; f < cnt * K3; f += kBlock) {
        const int gi = f / K3, q = f - gi * K3;
        float m = adam.m_sh[b0 + f], v = adam.v_sh[b0 + f];
        adam.sh[b0 + f] = adam_update(sh_s[gi * KP + q], gsh_s[gi * KP + q], m, v,
                                      q < 3 ? adam.lr_sh_dc : adam.lr_sh_rest, adam);
        adam.m_sh[b0 + f] = m;
        adam.v_sh[b0 + f] = v;
      }
    }
    return;
  }
  if constexpr (GQ) {
    // decode the accumulators, add this sub-batch's gradients, and quantise
    // the sums with the block's new scales
    const int64_t qb = blk >> 1;
    const int64_t nqb = (g.N + kGqBlock - 1) / kGqBlock;
    constexpr int kW[4] = {3, 4, 3, 1};  // widths of the per-thread attributes
    constexpr int kOff[4] = {0, 3, 7, 10};
    float old[kGqAttr];
#pragma unroll
    for (int a = 0; a < kGqAttr; ++a) old[a] = gqa.first ? 0.0f : gqa.scale[a * nqb + qb];
    float vmax[kGqAttr] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    if (valid) {
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int i = 0; i < kW[a]; ++i) {
          float x = gx[kOff[a] + i];
          if (!gqa.first) x += (float)gqa.code[a][kW[a] * n + i] * old[a];
          gx[kOff[a] + i] = x;
          vmax[a] = fmaxf(vmax[a], fabsf(x));
        }
    }
    // the block's SH codes: DC [128][3] and higher [128][K3-3] int16, each
    // contiguous and 16-byte aligned for a full block.  A full block copies
    // them as they are into shared memory (the SH staging area: the
    // coefficients are not needed after the camera walk) with every 16-byte
    // load in flight, and each thread then adds its own Gaussian's row, so no
    // code needs an index division; the ragged block goes word by word.
    constexpr int kDcV = kBlock * 3 * 2 / 16;
    constexpr int kRestV = kBlock * (K3 - 3) * 2 / 16;
    constexpr int kPerV = (kDcV + kRestV + kBlock - 1) / kBlock;
    constexpr int kDcN = kBlock * 3;
    const bool vec = cnt == kBlock;
    int16_t* code_s = reinterpret_cast<int16_t*>(sh_s);  // DC [kBlock][3], then higher [kBlock][K3 - 3]
    if (vec) {
      if (!gqa.first) {
        const int4* dc4 = reinterpret_cast<const int4*>(gqa.code[4] + 3 * n0);
        const int4* rest4 = reinterpret_cast<const int4*>(gqa.code[5] + (K3 - 3) * n0);
        int4* cs4 = reinterpret_cast<int4*>(code_s);
        int4 buf[kPerV];
#pragma unroll
        for (int r = 0; r < kPerV; ++r) {
          const int v = threadIdx.x + r * kBlock;
          if (v < kDcV) buf[r] = dc4[v];
          else if (v < kDcV + kRestV) buf[r] = rest4[v - kDcV];
        }
#pragma unroll
        for (int r = 0; r < kPerV; ++r) {
          const int v = threadIdx.x + r * kBlock;
          if (v < kDcV + kRestV) cs4[v] = buf[r];
        }
        __syncthreads();
      }
      float* gr = gsh_s + threadIdx.x * KP;
#pragma unroll
      for (int q = 0; q < K3; ++q) {
        float x = gr[q];
        if (!gqa.first) {
          const int16_t c = q < 3 ? code_s[3 * threadIdx.x + q] : code_s[kDcN + (K3 - 3) * threadIdx.x + (q - 3)];
          x = __fadd_rn(x, __fmul_rn((float)c, q < 3 ? old[4] : old[5]));
        }
        gr[q] = x;
        if (q < 3) vmax[4] = fmaxf(vmax[4], fabsf(x)); else vmax[5] = fmaxf(vmax[5], fabsf(x));
      }
    } else {
      for (int f = threadIdx.x; f < cnt * K3; f += kBlock) {
        const int gi = f / K3, q = f - gi * K3;
        const int64_t m = n0 + gi;
        float x = gsh_s[gi * KP + q];
        if (!gqa.first)
          x += q < 3 ? (float)gqa.code[4][3 * m + q] * old[4] : (float)gqa.code[5][(K3 - 3) * m + (q - 3)] * old[5];
        gsh_s[gi * KP + q] = x;
        if (q < 3) vmax[4] = fmaxf(vmax[4], fabsf(x)); else vmax[5] = fmaxf(vmax[5], fabsf(x));
      }
    }
    gq_cta_max(vmax, s_gq_wmax, s_gq_amax);
    float scale[kGqAttr], iscale[kGqAttr];
    gq_exchange(s_gq_amax, scale);  // the cluster barrier also orders the gsh_s updates above
#pragma unroll
    for (int a = 0; a < kGqAttr; ++a) iscale[a] = scale[a] > 0.0f ? 1.0f / scale[a] : 0.0f;
    if (valid) {
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int i = 0; i < kW[a]; ++i) gqa.code[a][kW[a] * n + i] = gq_code(gx[kOff[a] + i], iscale[a]);
    }
    if (vec) {
      // each thread quantises its own row into the shared code layout, then
      // 16-byte stores of eight codes each, the same vectors as the loads
      const float* gr = gsh_s + threadIdx.x * KP;
#pragma unroll
      for (int q = 0; q < K3; ++q) {
        const int16_t c = gq_code(gr[q], q < 3 ? iscale[4] : iscale[5]);
        if (q < 3) code_s[3 * threadIdx.x + q] = c; else code_s[kDcN + (K3 - 3) * threadIdx.x + (q - 3)] = c;
      }
      __syncthreads();
      int4* dc4 = reinterpret_cast<int4*>(gqa.code[4] + 3 * n0);
      int4* rest4 = reinterpret_cast<int4*>(gqa.code[5] + (K3 - 3) * n0);
      const int4* cs4 = reinterpret_cast<const int4*>(code_s);
      for (int v = threadIdx.x; v < kDcV + kRestV; v += kBlock) {
        if (v < kDcV) dc4[v] = cs4[v]; else rest4[v - kDcV] = cs4[v];
      }
    } else {
      for (int f = threadIdx.x; f < cnt * K3; f += kBlock) {
        const int gi = f / K3, q = f - gi * K3;
        const int64_t m = n0 + gi;
        const float x = gsh_s[gi * KP + q];
        if (q < 3) gqa.code[4][3 * m + q] = gq_code(x, iscale[4]);
        else gqa.code[5][(K3 - 3) * m + (q - 3)] = gq_code(x, iscale[5]);
      }
    }
    if ((blk & 1) == 0 && threadIdx.x < kGqAttr) {
      float sc = 0.0f;
#pragma unroll
      for (int a = 0; a < kGqAttr; ++a)
        if (a == (int)threadIdx.x) sc = scale[a];
      gqa.scale[threadIdx.x * nqb + qb] = sc;
    }
    return;
  }
  // write-back of the warp's own rows of the SH gradient block (16-byte
  // stores for a full warp; its lanes wrote the rows, so a warp barrier
  // suffices)
  __syncwarp();
  float* dst = v_sh + (n0 + 32 * warp) * K3;
  if (wrows == 32) {
    for (int v = lane; v < 32 * K3 / 4; v += 32) {
      float e[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        int gi, q;
        sh_word<K3>(v, u, gi, q);
        e[u] = gsh_w[gi * KP + q];
      }
      reinterpret_cast<float4*>(dst)[v] = make_float4(e[0], e[1], e[2], e[3]);
    }
  } else {
    for (int f = lane; f < wrows * K3; f += 32) {
      const int gi = f / K3, q = f - gi * K3;
      dst[f] = gsh_w[gi * KP + q];
    }
  }
}

template <int DEG, bool ADAM, bool GQ>
ss_status launch_pbwd(const Geo& g, cudaStream_t st, const float* cams, const float* means, const float* quats,
                      const float* scales, const float* sh, const uint32_t* mask, const int64_t* block_off,
                      const float* v_screen, float* v_means, float* v_quats, float* v_scales, float* v_opacities,
                      float* v_sh, const float* opacities, const AdamArgs& adam, const GqArgs& gqa) {
  const size_t smem = 2 * sizeof(float) * kBlock * sh_stride<DEG>();
  auto kernel = k_project_bwd<DEG, ADAM, GQ>;
  ss_status s = cuda_status(cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem),
                            "smem attr");
  if (s) return s;
  const int64_t ahead = wave_blocks(kernel, kBlock, smem);
  if constexpr (!GQ) {
    kernel<<<(unsigned)g.blocks_per_cam, kBlock, smem, st>>>(g, cams, means, quats, scales, sh, mask, block_off,
                                                              v_screen, v_means, v_quats, v_scales, v_opacities, v_sh,
                                                              opacities, adam, ahead, gqa);
    return cuda_status(cudaGetLastError(), "project bwd");
  } else {
    // clusters of two CTAs (one quantisation block of 256 Gaussians); an odd
    // block count gets one more CTA, which holds no Gaussians
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(g.blocks_per_cam + (g.blocks_per_cam & 1)));
    cfg.blockDim = dim3(kBlock);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cuda_status(cudaLaunchKernelEx(&cfg, kernel, g, cams, means, quats, scales, sh, mask, block_off, v_screen,
                                          v_means, v_quats, v_scales, v_opacities, v_sh, opacities, adam, ahead, gqa),
                       "project bwd (grad-quant)");
  }
}

template <bool ADAM, bool GQ>
ss_status dispatch_pbwd(const Geo& g, cudaStream_t st, const float* cams, const float* means, const float* quats,
                        const float* scales, const float* sh, const uint32_t* mask, const int64_t* block_off,
                        const float* v_screen, float* v_means, float* v_quats, float* v_scales, float* v_opacities,
                        float* v_sh, const float* opacities, const AdamArgs& adam, const GqArgs& gqa = GqArgs{}) {
  switch (g.deg) {
    case 0: return launch_pbwd<0, ADAM, GQ>(g, st, cams, means, quats, scales, sh, mask, block_off, v_screen,
                                            v_means, v_quats, v_scales, v_opacities, v_sh, opacities, adam, gqa);
    case 1: return launch_pbwd<1, ADAM, GQ>(g, st, cams, means, quats, scales, sh, mask, block_off, v_screen,
                                            v_means, v_quats, v_scales, v_opacities, v_sh, opacities, adam, gqa);
    case 2: return launch_pbwd<2, ADAM, GQ>(g, st, cams, means, quats, scales, sh, mask, block_off, v_screen,
                                            v_means, v_quats, v_scales, v_opacities, v_sh, opacities, adam, gqa);
    default: return launch_pbwd<3, ADAM, GQ>(g, st, cams, means, quats, scales, sh, mask, block_off, v_screen,
                                             v_means, v_quats, v_scales, v_opacities, v_sh, opacities, adam, gqa);
  }
}

}  // namespace ss

using namespace ss;

extern "C" ss_status ss_project_bwd(const ss_dims* dims, const float* cams, const float* means, const float* quats,
                                    const float* scales, const float* opacities, const float* sh,
                                    const uint32_t* mask, const int64_t* block_off, const float* v_screen,
                                    float* v_means, float* v_quats, float* v_scales, float* v_opacities, float* v_sh,
                                    void* stream) {
  if (!dims_ok(dims)) return invalid("dims");
  const Geo g = geometry(*dims);
  if (g.N == 0) return SS_OK;
  if (!cams || !means || !quats || !scales || !sh || !mask || !block_off || !v_screen) return invalid("null input");
  if (!v_means || !v_quats || !v_scales || !v_opacities || !v_sh) return invalid("null output");
  if (((uintptr_t)quats & 15) || ((uintptr_t)mask & 15) || ((uintptr_t)v_quats & 15) ||
      ((uintptr_t)v_screen & 15) || ((uintptr_t)sh & 15) || ((uintptr_t)v_sh & 15))
    return invalid("quats, mask, v_quats, v_screen, sh and v_sh must be 16-byte aligned");
  cudaStream_t st = as_stream(stream);
  return dispatch_pbwd<false, false>(g, st, cams, means, quats, scales, sh, mask, block_off, v_screen, v_means,
                                     v_quats, v_scales, v_opacities, v_sh, opacities, AdamArgs{});
}

extern "C" ss_status ss_project_bwd_adam(const ss_dims* dims, const float* cams, float* means, float* quats,
                                         float* log_scales, float* scales, float* logit_opacities, float* opacities,
                                         float* sh, const uint32_t* mask, const int64_t* block_off,
                                         const float* v_screen, const ss_adam_state* state, const ss_adam* hp,
                                         void* stream) {
  if (!dims_ok(dims)) return invalid("dims");
  const Geo g = geometry(*dims);
  if (g.N == 0) return SS_OK;
  if (!state || !hp) return invalid("null state or hyper-parameters");
  if (!cams || !means || !quats || !log_scales || !scales || !logit_opacities || !opacities || !sh || !mask ||
      !block_off || !v_screen)
    return invalid("null input");
  const ss_adam_state& S = *state;
  if (!S.m_means || !S.v_means || !S.m_quats || !S.v_quats || !S.m_scales || !S.v_scales || !S.m_opacities ||
      !S.v_opacities || !S.m_sh || !S.v_sh)
    return invalid("null optimizer state");
  if (((uintptr_t)quats & 15) || ((uintptr_t)mask & 15) || ((uintptr_t)v_screen & 15) || ((uintptr_t)sh & 15) ||
      ((uintptr_t)S.m_sh & 15) || ((uintptr_t)S.v_sh & 15))
    return invalid("quats, mask, v_screen, sh and the SH moments must be 16-byte aligned");
  if (hp->step < 1) return invalid("adam step must be >= 1");
  AdamArgs a{};
  a.m_means = S.m_means; a.v_means = S.v_means; a.m_quats = S.m_quats; a.v_quats = S.v_quats;
  a.m_scales = S.m_scales; a.v_scales = S.v_scales; a.m_opac = S.m_opacities; a.v_opac = S.v_opacities;
  a.m_sh = S.m_sh; a.v_sh = S.v_sh;
  a.means = means; a.quats = quats; a.log_scales = log_scales; a.scales = scales; a.logit_opac = logit_opacities;
  a.opac = opacities; a.sh = sh;
  a.lr_means = hp->lr_means; a.lr_quats = hp->lr_quats; a.lr_scales = hp->lr_scales;
  a.lr_opac = hp->lr_opacities; a.lr_sh_dc = hp->lr_sh_dc; a.lr_sh_rest = hp->lr_sh_rest;
  a.b1 = hp->beta1; a.b2 = hp->beta2; a.eps = hp->eps;
  a.ibc1 = (float)(1.0 / (1.0 - std::pow((double)hp->beta1, (double)hp->step)));
  a.ibc2s = (float)(1.0 / std::sqrt(1.0 - std::pow((double)hp->beta2, (double)hp->step)));
  cudaStream_t st = as_stream(stream);
  return dispatch_pbwd<true, false>(g, st, cams, means, quats, scales, sh, mask, block_off, v_screen, nullptr,
                                    nullptr, nullptr, nullptr, nullptr, opacities, a);
}

extern "C" ss_status ss_project_bwd_gq(const ss_dims* dims, const float* cams, const float* means, const float* quats,
                                       const float* scales, const float* opacities, const float* sh,
                                       const uint32_t* mask, const int64_t* block_off, const float* v_screen,
                                       const ss_gq_accum* acc, int first, void* stream) {
  if (!dims_ok(dims)) return invalid("dims");
  const Geo g = geometry(*dims);
  if (g.N == 0) return SS_OK;
  if (!cams || !means || !quats || !scales || !sh || !mask || !block_off || !v_screen) return invalid("null input");
  if (!acc || !acc->means || !acc->quats || !acc->scales || !acc->opacities || !acc->sh_dc || !acc->block_scale ||
      (g.deg > 0 && !acc->sh_rest))
    return invalid("null accumulator");
  if (((uintptr_t)quats & 15) || ((uintptr_t)mask & 15) || ((uintptr_t)v_screen & 15) || ((uintptr_t)sh & 15))
    return invalid("quats, mask, v_screen and sh must be 16-byte aligned");
  if (((uintptr_t)acc->sh_dc & 15) || ((uintptr_t)acc->sh_rest & 15))
    return invalid("the SH code arrays must be 16-byte aligned");
  GqArgs q{};
  q.code[0] = acc->means;
  q.code[1] = acc->quats;
  q.code[2] = acc->scales;
  q.code[3] = acc->opacities;
  q.code[4] = acc->sh_dc;
  q.code[5] = acc->sh_rest;
  q.scale = acc->block_scale;
  q.first = first ? 1 : 0;
  cudaStream_t st = as_stream(stream);
  return dispatch_pbwd<false, true>(g, st, cams, means, quats, scales, sh, mask, block_off, v_screen, nullptr,
                                    nullptr, nullptr, nullptr, nullptr, opacities, AdamArgs{}, q);
}
