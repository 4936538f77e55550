// Host builder of the LVSA per-query-frame KV frame lists.
//
// "LVSA: Training-Free Sparse Attention for Long Video Diffusion":
//   A(t) = G_s U W(t)                       gist.science technical summary, sec. 2 "Core Mechanism"
//   G = C - W anchors, spacing ~ T/(C-W)    techwalker article, section 二
//   anchors shift one frame per step mod T  techwalker article, section 三
//   window extension until |A(t)| = C       gist.science summary "Expanded Adaptive Windows";
//                                           techwalker article, section 二
//
// Formulation used here (closed form, O(T + T*C) per call): instead of growing
// the window turn by turn, count the non-anchor frames on each side of the
// window with a prefix sum and split the missing budget k = C - |G U window|
// between the sides: the right side takes ceil(k/2) and the left floor(k/2);
// a side with fewer free frames than its share gives the rest to the other
// side.  That is exactly what alternating right/left turns of one new
// non-anchor frame each produce.  The new window ends are the positions of
// the r-th free frame right of the window and the l-th free frame left of it,
// read from an index of free-frame positions.  Each row is then written by
// merging the sorted anchors with that interval.
#include <stdint.h>
#include <stddef.h>

#include <algorithm>
#include <vector>

#include "lvsa.h"

namespace {

bool params_ok(int T, int C, int W, long long step) {
  return T >= 1 && C >= 1 && W >= 1 && W <= C && step >= 0;
}

// Anchor frames of step `step`, ascending.  Requires 0 < G < T.
void anchor_frames(int T, int G, long long step, std::vector<int32_t>& a) {
  a.resize(G);
  const long long s = step % T;
  for (int k = 0; k < G; ++k) {
    const long long off = (static_cast<long long>(k) * T) / G;  // floor(k*T/G)
    a[k] = static_cast<int32_t>((s + off) % T);
  }
  std::sort(a.begin(), a.end());
}

}  // namespace

extern "C" lvsa_status lvsa_build_anchors(int T, int C, int W, long long step, int32_t* out,
                                          size_t out_capacity, int* out_G) {
  if (!params_ok(T, C, W, step)) return LVSA_ERR_INVALID_ARG;
  const int G = (C >= T) ? 0 : C - W;
  if (out_G) *out_G = G;
  if (G == 0) return LVSA_OK;
  if (out == nullptr || out_capacity < static_cast<size_t>(G)) return LVSA_ERR_BUFFER_TOO_SMALL;
  std::vector<int32_t> a;
  anchor_frames(T, G, step, a);
  std::copy(a.begin(), a.end(), out);
  return LVSA_OK;
}

extern "C" lvsa_status lvsa_build_frame_lists(int T, int C, int W, long long step, int32_t* out,
                                              size_t out_capacity, int* out_L) {
  if (!params_ok(T, C, W, step)) return LVSA_ERR_INVALID_ARG;
  const int L = std::min(C, T);
  if (out_L) *out_L = L;
  if (out == nullptr || out_capacity < static_cast<size_t>(T) * static_cast<size_t>(L))
    return LVSA_ERR_BUFFER_TOO_SMALL;

  if (C >= T) {  // the budget covers the whole video: dense rows
    for (int t = 0; t < T; ++t)
      for (int f = 0; f < T; ++f) out[static_cast<size_t>(t) * L + f] = f;
    return LVSA_OK;
  }

  const int G = C - W;
  std::vector<int32_t> anchors;
  if (G > 0) anchor_frames(T, G, step, anchors);

  std::vector<uint8_t> is_anchor(T, 0);
  for (int32_t f : anchors) is_anchor[f] = 1;
  // free_before[i] = number of non-anchor frames in [0, i); free_pos[j] = j-th non-anchor frame
  std::vector<int> free_before(T + 1, 0);
  std::vector<int> free_pos;
  free_pos.reserve(T);
  for (int f = 0; f < T; ++f) {
    free_before[f + 1] = free_before[f] + (is_anchor[f] ? 0 : 1);
    if (!is_anchor[f]) free_pos.push_back(f);
  }

  std::vector<int32_t> row;
  row.reserve(C);
  for (int t = 0; t < T; ++t) {
    // window of W frames, lo = t - W/2, moved inside [0, T-1]
    int lo = std::min(std::max(t - W / 2, 0), T - W);
    int hi = lo + W - 1;

    const int free_in_window = free_before[hi + 1] - free_before[lo];
    const int missing = C - (G + free_in_window);  // >= 0 since G + W = C
    const int free_right = free_before[T] - free_before[hi + 1];
    const int free_left = free_before[lo];
    int take_r = (missing + 1) / 2;
    int take_l = missing / 2;
    if (take_r > free_right) {
      take_l += take_r - free_right;
      take_r = free_right;
    } else if (take_l > free_left) {
      take_r += take_l - free_left;
      take_l = free_left;
    }
    if (take_r > 0) hi = free_pos[free_before[hi + 1] + take_r - 1];
    if (take_l > 0) lo = free_pos[free_before[lo] - take_l];

    // merge: anchors below lo, the interval [lo, hi], anchors above hi
    row.clear();
    size_t ai = 0;
    while (ai < anchors.size() && anchors[ai] < lo) row.push_back(anchors[ai++]);
    for (int f = lo; f <= hi; ++f) row.push_back(f);
    while (ai < anchors.size() && anchors[ai] <= hi) ++ai;
    while (ai < anchors.size()) row.push_back(anchors[ai++]);
    if (static_cast<int>(row.size()) != L) return LVSA_ERR_INVALID_ARG;  // cannot happen: |G U [lo,hi]| = C
    std::copy(row.begin(), row.end(), out + static_cast<size_t>(t) * L);
  }
  return LVSA_OK;
}
