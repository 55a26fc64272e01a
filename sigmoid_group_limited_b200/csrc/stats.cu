// stats.cu - routing statistics from the expert counts (load monitoring).
//
// Page "Ling-3.0-flash-VL：层级化稀疏路由大模型硬核解析" (sheratonhq.com/news/113555),
// sec. 4.1: watch the routing entropy H = -sum_e p_e log2 p_e of the expert
// selection frequencies, and count experts that are never selected. Page
// "Ling-3.0-flash-VL MoE sparse routing" (lqnn.cn/news/282163), sec. 3 step 3:
// the per-expert bias exists to keep those loads balanced.
//
// One CTA of 1024 threads (E <= 1024), thread e owns expert e. Integer
// totals are order-free; the entropy terms are added in a fixed tree order,
// so the result does not depend on scheduling.
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "internal.h"
#include "ptx.cuh"

namespace sgl {
namespace {

__global__ void __launch_bounds__(1024) route_stats(int E, const int32_t* __restrict__ counts,
                                                    double* __restrict__ stats) {
  pdl_trigger();
  pdl_wait();  // the counts come from an earlier kernel
  __shared__ long long s_tot;
  __shared__ int s_max, s_idle;
  __shared__ double term[1024];
  const int e = threadIdx.x;
  if (e == 0) {
    s_tot = 0;
    s_max = 0;
    s_idle = 0;
  }
  __syncthreads();
  const int c = e < E ? max(counts[e], 0) : 0;
  if (e < E) {
    atomicAdd(reinterpret_cast<unsigned long long*>(&s_tot), static_cast<unsigned long long>(c));
    atomicMax(&s_max, c);
    if (c == 0) atomicAdd(&s_idle, 1);
  }
  __syncthreads();
  const double tot = static_cast<double>(s_tot);
  double t = 0.0;
  if (e < E && c > 0 && tot > 0.0) {
    const double pe = c / tot;
    t = -pe * log2(pe);
  }
  term[e] = t;
  __syncthreads();
  for (int stride = 512; stride > 0; stride >>= 1) {  // fixed pairwise order
    if (e < stride) term[e] += term[e + stride];
    __syncthreads();
  }
  if (e == 0) {
    const double H = term[0];
    const double mean = tot / E;
    stats[0] = H;
    stats[1] = E > 1 ? H / log2(static_cast<double>(E)) : 0.0;
    stats[2] = static_cast<double>(s_max);
    stats[3] = mean;
    stats[4] = mean > 0.0 ? s_max / mean : 0.0;
    stats[5] = static_cast<double>(s_idle);
    stats[6] = tot;
  }
}

}  // namespace

cudaError_t launch_route_stats(const moe_cfg& c, const int32_t* counts, double* stats,
                               cudaStream_t s) {
  return launch_pdl(route_stats, dim3(1), dim3(1024), 0, s, c.E, counts, stats);
}

}  // namespace sgl
