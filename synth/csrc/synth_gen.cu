// Device twin of the seeded input generator in synth/{philox,normal,workload}.py.
//
// It evaluates the same integer Philox4x32-10 function and the same
// Box-Muller doubles (series logarithm, sine and cosine written with
// correctly rounded, unfused double operations in the same order as the
// numpy code), so caches filled here are bit-identical to the slices the host
// regenerates. It draws inputs only; it holds no attention arithmetic and is
// built as its own library, separate from the SAGA library.
#include <cuda_runtime.h>
#include <stdint.h>

namespace {

constexpr uint32_t kM0 = 0xD2511F53u, kM1 = 0xCD9E8D57u;
constexpr uint32_t kW0 = 0x9E3779B9u, kW1 = 0xBB67AE85u;
constexpr int kNAtanh = 12, kNTrig = 13, kMaxD = 128;

struct Consts {
  double atanh_c[kNAtanh];
  double sin_c[kNTrig];
  double cos_c[kNTrig];
  double ln2, half_pi, sqrt2;
  double u[kMaxD];          // unit direction of planted keys
  double plant_scale, plant_noise;
};

struct FillArgs {
  void *out;
  int64_t stride_b, stride_h;   // elements; token stride = d
  int64_t T;                    // tokens filled per (b, h)
  int32_t B, H, d, dtype;       // dtype 0 fp32, 1 bf16
  uint32_t seed, tensor, layer;
  uint32_t plant, plant_tensor, plant_head_offset, plant_thresh;
};

__device__ __forceinline__ void philox(uint32_t c[4], uint32_t k0, uint32_t k1) {
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    const uint64_t p0 = static_cast<uint64_t>(kM0) * c[0];
    const uint64_t p1 = static_cast<uint64_t>(kM1) * c[2];
    const uint32_t n0 = static_cast<uint32_t>(p1 >> 32) ^ c[1] ^ k0;
    const uint32_t n1 = static_cast<uint32_t>(p1);
    const uint32_t n2 = static_cast<uint32_t>(p0 >> 32) ^ c[3] ^ k1;
    const uint32_t n3 = static_cast<uint32_t>(p0);
    c[0] = n0; c[1] = n1; c[2] = n2; c[3] = n3;
    if (r != 9) { k0 += kW0; k1 += kW1; }
  }
}

__device__ __forceinline__ double horner(const double *c, int n, double t) {
  double p = c[n - 1];
  for (int k = n - 2; k >= 0; --k) {
    p = __dmul_rn(p, t);
    p = __dadd_rn(p, c[k]);
  }
  return p;
}

__device__ double ln_u1(uint32_t x, const Consts &k) {
  const double n = static_cast<double>(x) + 1.0;   // exact
  int e;
  double m = frexp(n, &e);                          // exact
  m = __dmul_rn(m, 2.0);
  double ef = static_cast<double>(e) - 1.0;
  if (m > k.sqrt2) { m = __dmul_rn(m, 0.5); ef = ef + 1.0; }
  const double s = __ddiv_rn(__dadd_rn(m, -1.0), __dadd_rn(m, 1.0));
  const double s2 = __dmul_rn(s, s);
  const double p = horner(k.atanh_c, kNAtanh, s2);
  const double lnm = __dmul_rn(__dmul_rn(2.0, s), p);
  return __dadd_rn(__dmul_rn(ef - 32.0, k.ln2), lnm);
}

__device__ void sincos_2pi(uint32_t x, const Consts &k, double &sn, double &cs) {
  const uint32_t quad = x >> 30;
  const double f = __dmul_rn(static_cast<double>(x & 0x3FFFFFFFu), 0x1p-30);
  const double th = __dmul_rn(f, k.half_pi);
  const double t = __dmul_rn(th, th);
  const double s = __dmul_rn(th, horner(k.sin_c, kNTrig, t));
  const double c = horner(k.cos_c, kNTrig, t);
  switch (quad) {
    case 0: sn = s; cs = c; break;
    case 1: sn = c; cs = -s; break;
    case 2: sn = -s; cs = -c; break;
    default: sn = -c; cs = s; break;
  }
}

__device__ __forceinline__ void box_muller(uint32_t xa, uint32_t xb, const Consts &k, double &z0,
                                           double &z1) {
  const double r = __dsqrt_rn(__dmul_rn(-2.0, ln_u1(xa, k)));
  double sn, cs;
  sincos_2pi(xb, k, sn, cs);
  z0 = __dmul_rn(r, cs);
  z1 = __dmul_rn(r, sn);
}

__device__ __forceinline__ uint16_t to_bf16(float f) {
  const uint32_t b = __float_as_uint(f);
  return static_cast<uint16_t>((b + 0x7FFFu + ((b >> 16) & 1u)) >> 16);
}

// One thread per Philox block (four consecutive elements of one (b, h) row).
__global__ void fill_kernel(const FillArgs a, const Consts k) {
  const int64_t blocks_per_row = a.T * a.d / 4;
  const int64_t gid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t total = blocks_per_row * a.B * a.H;
  if (gid >= total) return;
  const int64_t m = gid % blocks_per_row;
  const int64_t bh = gid / blocks_per_row;
  const uint32_t h = static_cast<uint32_t>(bh % a.H), b = static_cast<uint32_t>(bh / a.H);
  const uint32_t key1 = (a.tensor & 0xFFu) | ((a.layer & 0xFFu) << 8);
  uint32_t c[4] = {static_cast<uint32_t>(m), h, b, 0u};
  philox(c, a.seed, key1);
  double z[4];
  box_muller(c[0], c[1], k, z[0], z[1]);
  box_muller(c[2], c[3], k, z[2], z[3]);
  const int64_t e0 = m * 4;
  const int64_t t = e0 / a.d;             // all four elements share a token (d % 4 == 0)
  const int i0 = static_cast<int>(e0 % a.d);
  if (a.plant) {
    const uint32_t pkey1 = (a.plant_tensor & 0xFFu) | ((a.layer & 0xFFu) << 8);
    uint32_t pc[4] = {static_cast<uint32_t>(t >> 2), h + a.plant_head_offset, b, 0u};
    philox(pc, a.seed, pkey1);
    if (pc[t & 3] < a.plant_thresh) {
#pragma unroll
      for (int e = 0; e < 4; ++e)
        z[e] = __dadd_rn(__dmul_rn(k.plant_scale, k.u[i0 + e]), __dmul_rn(k.plant_noise, z[e]));
    }
  }
  const int64_t off = b * a.stride_b + h * a.stride_h + e0;
  if (a.dtype == 0) {
    float4 v = make_float4(__double2float_rn(z[0]), __double2float_rn(z[1]),
                           __double2float_rn(z[2]), __double2float_rn(z[3]));
    *reinterpret_cast<float4 *>(static_cast<float *>(a.out) + off) = v;
  } else {
    ushort4 v;
    v.x = to_bf16(__double2float_rn(z[0]));
    v.y = to_bf16(__double2float_rn(z[1]));
    v.z = to_bf16(__double2float_rn(z[2]));
    v.w = to_bf16(__double2float_rn(z[3]));
    *reinterpret_cast<ushort4 *>(static_cast<uint16_t *>(a.out) + off) = v;
  }
}

}  // namespace

extern "C" {

// Fill out[b][h][t][i] for b < B, h < H, t < T, i < d (d % 4 == 0, d <= 128).
// consts: host array laid out as struct Consts (see synth/device.py).
// Returns a cudaError_t value (0 on success).
int synth_fill(void *out, int64_t stride_b, int64_t stride_h, int64_t T, int32_t B, int32_t H,
               int32_t d, int32_t dtype, uint32_t seed, uint32_t tensor, uint32_t layer,
               uint32_t plant, uint32_t plant_tensor, uint32_t plant_head_offset,
               uint32_t plant_thresh, const double *consts, void *stream) {
  if (d % 4 != 0 || d > kMaxD || out == nullptr || consts == nullptr) return 1;
  FillArgs a{out, stride_b, stride_h, T, B, H, d, dtype, seed, tensor, layer,
             plant, plant_tensor, plant_head_offset, plant_thresh};
  Consts k;
  const double *c = consts;
  for (int i = 0; i < kNAtanh; ++i) k.atanh_c[i] = *c++;
  for (int i = 0; i < kNTrig; ++i) k.sin_c[i] = *c++;
  for (int i = 0; i < kNTrig; ++i) k.cos_c[i] = *c++;
  k.ln2 = *c++; k.half_pi = *c++; k.sqrt2 = *c++;
  for (int i = 0; i < kMaxD; ++i) k.u[i] = *c++;
  k.plant_scale = *c++; k.plant_noise = *c++;
  const int64_t total = T * d / 4 * B * H;
  if (total == 0) return 0;
  const int threads = 256;
  const int64_t grid = (total + threads - 1) / threads;
  fill_kernel<<<static_cast<unsigned>(grid), threads, 0, static_cast<cudaStream_t>(stream)>>>(a, k);
  return static_cast<int>(cudaGetLastError());
}

}  // extern "C"
