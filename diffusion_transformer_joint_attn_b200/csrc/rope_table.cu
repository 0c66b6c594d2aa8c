// Three-axis rotary embedding table: cos/sin of pos[n][a] * theta^(-2i/d_a)
// for every token n and channel pair j (axis a, index i inside the axis).
#include <cmath>

#include "launch.h"

namespace dit {

struct RopeAxes {
  int width[3];
};

__global__ void rope_table_kernel(const int32_t* __restrict__ pos, int N, int pairs, RopeAxes axes,
                                  double log_theta, float* __restrict__ out_cos, float* __restrict__ out_sin) {
  const long long idx = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= static_cast<long long>(N) * pairs) return;
  const int n = static_cast<int>(idx / pairs);
  const int j = static_cast<int>(idx % pairs);
  // locate the axis slice that owns pair j
  int a = 0, first = 0;
  while (a < 2 && j >= first + axes.width[a] / 2) {
    first += axes.width[a] / 2;
    ++a;
  }
  const int i = j - first;
  const double omega = exp(-2.0 * i / axes.width[a] * log_theta);
  const double phi = static_cast<double>(pos[n * 3 + a]) * omega;
  double s, c;
  sincos(phi, &s, &c);
  out_cos[idx] = static_cast<float>(c);
  out_sin[idx] = static_cast<float>(s);
}

cudaError_t launch_rope_table(const RopeTableArgs& a, cudaStream_t s) {
  const int pairs = a.D / 2;
  const long long total = static_cast<long long>(a.N) * pairs;
  const int threads = 256;
  const long long blocks = (total + threads - 1) / threads;
  RopeAxes axes{{a.axes[0], a.axes[1], a.axes[2]}};
  rope_table_kernel<<<static_cast<unsigned>(blocks), threads, 0, s>>>(a.pos, a.N, pairs, axes, std::log(a.theta),
                                                                      a.cos, a.sin);
  return cudaGetLastError();
}

}  // namespace dit
