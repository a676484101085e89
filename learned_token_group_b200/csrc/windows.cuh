// STGA window geometry shared by the forward and backward attention kernels.
//
// "Spatial-Temporal Group Attention" (MoGA paper summary, section 3.4): fixed
// local windows of (wt, wh, ww) latent tokens over the (T, Hg, Wg) grid,
// anchored at the origin and clipped at the edges.  Windows are numbered with
// the temporal block outermost, then rows, then columns; window seg's tokens
// occupy positions [start, start + len) of the window order.
#pragma once

namespace moga {

struct WinGeom {
  int T, Hg, Wg, wt, wh, ww, nbh, nbw;  // nbh, nbw: windows per column / row of a frame
};

__device__ __forceinline__ void window_of(const WinGeom& g, int seg, int& start, int& len) {
  const int tb = seg / (g.nbh * g.nbw);
  const int hb = (seg / g.nbw) % g.nbh;
  const int wb = seg % g.nbw;
  const int t0 = tb * g.wt, h0 = hb * g.wh, w0 = wb * g.ww;
  const int et = min(g.wt, g.T - t0), eh = min(g.wh, g.Hg - h0), ew = min(g.ww, g.Wg - w0);
  start = t0 * g.Hg * g.Wg + et * (h0 * g.Wg + eh * w0);
  len = et * eh * ew;
}

}  // namespace moga
