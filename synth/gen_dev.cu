// Device build of the seeded synthetic-input generator (see gen_core.h).
// Produces the same bits as gen_host.c for the same arguments; it exists so
// that full-size step inputs can be regenerated on the GPU without a host
// round trip.  Compiled with -fmad=false so that no multiply-add is fused.
#include <cuda_runtime.h>
#include <stdint.h>

#include "gen_core.h"

namespace {

__global__ void fill_kernel(void* out, int dtype, int B, int L, int Hx, int d, int bs,
                            uint32_t step, uint32_t tensor, uint32_t k0, uint32_t k1,
                            double unit, double noise, const double* sharp, const double* dir,
                            const uint8_t* plant, double amp) {
  const uint64_t total = (uint64_t)B * L * Hx * d;
  const int nb = L / bs;
  for (uint64_t elem = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; elem < total;
       elem += (uint64_t)gridDim.x * blockDim.x) {
    uint64_t row = elem / ((uint64_t)Hx * d);
    int h = (int)((elem / d) % Hx);
    int c = (int)(elem % d);
    int b = (int)(row / L);
    int t = (int)(row % L);
    double sh = sharp ? sharp[h] : 1.0;
    double shift = 0.0;
    if (plant && dir && plant[((int64_t)b * Hx + h) * nb + t / bs])
      shift = amp * dir[((int64_t)b * Hx + h) * d + c];
    double x = syn_value(elem, step, tensor, k0, k1, unit, noise, sh, shift);
    float f = __double2float_rn(x);
    if (dtype == 1)
      ((float*)out)[elem] = f;
    else
      ((uint16_t*)out)[elem] = syn_f32_to_bf16(f);
  }
}

}  // namespace

// Device pointers for out, sharp, dir and plant.  Returns a cudaError_t value.
extern "C" int synth_fill_dev(void* out, int dtype, int B, int L, int Hx, int d, int bs,
                              uint32_t step, uint32_t tensor, uint64_t seed, double unit,
                              double noise, const double* sharp, const double* dir,
                              const uint8_t* plant, double amp, void* stream) {
  if (!out || B <= 0 || L <= 0 || Hx <= 0 || d <= 0 || bs <= 0 || L % bs)
    return (int)cudaErrorInvalidValue;
  uint64_t total = (uint64_t)B * L * Hx * d;
  uint64_t blocks = (total + 255) / 256;
  if (blocks > 148ull * 64) blocks = 148ull * 64;
  fill_kernel<<<(unsigned)blocks, 256, 0, (cudaStream_t)stream>>>(
      out, dtype, B, L, Hx, d, bs, step, tensor, (uint32_t)seed, (uint32_t)(seed >> 32), unit,
      noise, sharp, dir, plant, amp);
  return (int)cudaGetLastError();
}
