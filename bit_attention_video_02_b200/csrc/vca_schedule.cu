// vca_schedule.cu -- when a layer regroups its value tokens over a denoising
// run ("Nunchux AI Introduces VC-Attention...", abstract and section
// "V-Smooth 與 ExpCast-FP8": grouping only in the first 25 % of the steps, each
// permutation reused across 4 adjacent steps).  Host-only decision; the
// grouping itself is vca_cluster_permute.
#include "vca_host.h"

using namespace vca;

extern "C" int vca_schedule_regroup(int step, int total_steps, int reuse, float group_fraction) {
  if (total_steps < 1 || step < 0 || step >= total_steps || reuse < 1 || !(group_fraction > 0.0f) ||
      group_fraction > 1.0f)
    return fail(VCA_ERR_INVALID, "vca_schedule_regroup: bad arguments (step %d of %d, reuse %d, fraction %g)",
                step, total_steps, reuse, (double)group_fraction);
  if (step == 0) return 1;
  // step < fraction * total, compared in double so 0.25 * 50 = 12.5 admits step 12
  return ((double)step < (double)group_fraction * (double)total_steps && step % reuse == 0) ? 1 : 0;
}
