// Host-side launch planning shared by the kernels' launchers: plain C++,
// no CUDA, so that it can be compiled and checked on its own.
#pragma once

#include <algorithm>
#include <cstdint>

namespace hxq {

// Stream-K shares of a group's grid: G CTAs, layer i getting about
// G W[i] / sum W of them, at least 1 and at most W[i]; the CTAs left over
// (or taken back) go to (come from) the layers with the most (fewest)
// stages per CTA.
inline void group_shares(const int64_t* W, int n, int G, int* Gl) {
  int64_t Wt = 0;
  for (int i = 0; i < n; ++i) Wt += W[i];
  int sum = 0;
  for (int i = 0; i < n; ++i) {
    Gl[i] = (int)std::max<int64_t>(1, std::min<int64_t>(W[i], (int64_t)G * W[i] / Wt));
    sum += Gl[i];
  }
  while (sum < G) {  // W[i] / Gl[i] largest among the layers that can take one more
    int best = -1;
    for (int i = 0; i < n; ++i)
      if (Gl[i] < W[i] && (best < 0 || W[i] * Gl[best] > W[best] * Gl[i])) best = i;
    if (best < 0) break;
    ++Gl[best];
    ++sum;
  }
  while (sum > G) {  // W[i] / Gl[i] smallest among the layers that can give one up
    int best = -1;
    for (int i = 0; i < n; ++i)
      if (Gl[i] > 1 && (best < 0 || W[i] * Gl[best] < W[best] * Gl[i])) best = i;
    if (best < 0) break;
    --Gl[best];
    --sum;
  }
}

}  // namespace hxq
