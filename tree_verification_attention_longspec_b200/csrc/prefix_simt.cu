// Prefix partial attention on CUDA cores: one CTA per chunk, one thread per query row.
//
// The "Cached-Teil" of section 2C (LongSpec, gist.science summary): every tree
// query attends to its sequence's cached prefix with no mask. A chunk covers 256
// query rows of one kv head and a range of prefix keys; it leaves a partial
// softmax result (out normalised by its own sum, lse in the log2 domain) that the
// tree/combine kernel merges exactly.
//
// This is the plain SIMT formulation: keys and values are staged 32 at a time in
// shared memory as fp32, each thread keeps its row's running max, sum and output in
// registers and rescales once per 32-key tile.
#include "ls_device.cuh"

namespace ls {
namespace {

constexpr int kTileKeys = 32;
constexpr int kThreads = kUnitRows;  // one thread per row of the chunk

template <int D>
__global__ void __launch_bounds__(kThreads, 1) prefix_simt_kernel(PrefixArgs a) {
  extern __shared__ float smem[];
  float* qT = smem;                         // [D][256], pre-scaled by scale*log2(e)
  float* ks = qT + D * kThreads;            // [32][D]
  float* vs = ks + kTileKeys * D;           // [32][D]
  const Plan& p = a.p;
  const int t = threadIdx.x;
  const ChunkCoord c = locate_chunk(p, a.cu, blockIdx.x);
  if (!c.valid) return;  // grid larger than the device lengths: reported by the combine

  const int r = c.rgi * kUnitRows + t;
  const bool valid = r < p.rows;
  const int i = r / p.g, j = r % p.g;
  const uint16_t* qrow = a.q + ((size_t)(c.b * p.T + (valid ? i : 0)) * p.Hq + c.kh * p.g + j) * D;
  for (int cc = 0; cc < D; ++cc)
    qT[cc * kThreads + t] = valid ? bf16_to_f32(qrow[cc]) * p.scale_log2 : 0.f;

  float o[D];
#pragma unroll
  for (int cc = 0; cc < D; ++cc) o[cc] = 0.f;
  float m = -INFINITY, l = 0.f;

  for (int k0 = c.key_begin; k0 < c.key_end; k0 += kTileKeys) {
    const int n = min(kTileKeys, c.key_end - k0);
    __syncthreads();
    for (int e = t; e < kTileKeys * D; e += kThreads) {
      const int kk = e / D, cc = e % D;
      float kv = 0.f, vv = 0.f;
      if (kk < n) {
        const size_t row = ((size_t)(c.seq_offset + k0 + kk) * p.Hkv + c.kh) * D + cc;
        kv = bf16_to_f32(a.k_cache[row]);
        vv = bf16_to_f32(a.v_cache[row]);
      }
      ks[e] = kv;
      vs[e] = vv;
    }
    __syncthreads();

    float s[kTileKeys];
#pragma unroll
    for (int kk = 0; kk < kTileKeys; ++kk) s[kk] = 0.f;
#pragma unroll 2
    for (int cc = 0; cc < D; ++cc) {
      const float qv = qT[cc * kThreads + t];
#pragma unroll
      for (int kk = 0; kk < kTileKeys; ++kk) s[kk] = fmaf(qv, ks[kk * D + cc], s[kk]);
    }
    float mt = -INFINITY;
#pragma unroll
    for (int kk = 0; kk < kTileKeys; ++kk) {
      s[kk] = kk < n ? s[kk] : -INFINITY;
      mt = fmaxf(mt, s[kk]);
    }
    const float mn = fmaxf(m, mt);
    const float corr = exp2f(m - mn);  // first tile: exp2(-inf) = 0
    l *= corr;
#pragma unroll
    for (int cc = 0; cc < D; ++cc) o[cc] *= corr;
    m = mn;
#pragma unroll 1
    for (int kk = 0; kk < n; ++kk) {
      float pk = 0.f;
#pragma unroll
      for (int x = 0; x < kTileKeys; ++x) pk = (x == kk) ? s[x] : pk;
      pk = exp2f(pk - m);
      l += pk;
#pragma unroll
      for (int cc = 0; cc < D; ++cc) o[cc] = fmaf(pk, vs[kk * D + cc], o[cc]);
    }
  }

  if (valid) {
    const size_t slot = (size_t)blockIdx.x * kUnitRows + t;
    float lse2 = -INFINITY, inv = 0.f;
    if (l > 0.f) {
      lse2 = m + log2f(l);
      inv = 1.f / l;
    }
    a.lse_part[slot] = lse2;
    float4* dst = reinterpret_cast<float4*>(a.o_part + slot * D);
#pragma unroll
    for (int cc = 0; cc < D; cc += 4)
      dst[cc / 4] = make_float4(o[cc] * inv, o[cc + 1] * inv, o[cc + 2] * inv, o[cc + 3] * inv);
  }
  if (t == 0) a.chunk_status[blockIdx.x] = 0u;
}

template <int D>
cudaError_t launch_d(const PrefixArgs& a, cudaStream_t stream) {
  const size_t smem = (size_t)(D * kThreads + 2 * kTileKeys * D) * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(prefix_simt_kernel<D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  prefix_simt_kernel<D><<<a.p.n_chunks, kThreads, smem, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prefix_simt(const PrefixArgs& a, cudaStream_t stream) {
  if (a.p.n_chunks == 0) return cudaSuccess;
  return a.p.d == 64 ? launch_d<64>(a, stream) : launch_d<128>(a, stream);
}

}  // namespace ls
