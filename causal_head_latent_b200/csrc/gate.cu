// The channel-wise output gate as a stand-alone pass ("Gated MLA" page, "The
// channel-wise output gate"): out = sigmoid(G) (.) O element by element, in
// float32, one bfloat16 rounding.  The attention epilogues already fuse the
// gate; this pass serves gmla_gate_out when its caller hands over an ungated
// context.  HBM-bound: 16-byte loads and stores, a grid of a few CTAs per SM
// striding over the elements.
#include "internal.h"
#include "ptx.cuh"

namespace gmla {
namespace gate {

__global__ void __launch_bounds__(256) gate_kernel(const uint4 *__restrict__ O, const uint4 *__restrict__ G,
                                                   uint4 *__restrict__ out, size_t n8) {
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n8; i += (size_t)gridDim.x * blockDim.x) {
    const uint4 o = O[i], g = G[i];
    const uint32_t ow[4] = {o.x, o.y, o.z, o.w}, gw[4] = {g.x, g.y, g.z, g.w};
    uint32_t r[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float lo = bf16_to_f32(ow[e] & 0xFFFF) * sigmoidf_(bf16_to_f32(gw[e] & 0xFFFF));
      const float hi = bf16_to_f32(ow[e] >> 16) * sigmoidf_(bf16_to_f32(gw[e] >> 16));
      r[e] = pack_bf16x2(lo, hi);
    }
    out[i] = make_uint4(r[0], r[1], r[2], r[3]);
  }
}

}  // namespace gate

// n (a multiple of 8) elements; all three pointers 16-byte aligned.
int launch_gate(const uint16_t *O, const uint16_t *G, uint16_t *out, size_t n, cudaStream_t stream) {
  const size_t n8 = n / 8;
  if (n8 == 0) return 0;
  const size_t want = (n8 + 255) / 256;
  const unsigned grid = (unsigned)(want < (size_t)8 * num_sms() ? want : (size_t)8 * num_sms());
  gate::gate_kernel<<<grid, 256, 0, stream>>>(reinterpret_cast<const uint4 *>(O), reinterpret_cast<const uint4 *>(G),
                                             reinterpret_cast<uint4 *>(out), n8);
  return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

}  // namespace gmla
