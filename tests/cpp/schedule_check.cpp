// Host-side check of the Newton-Schulz list scheduler (schedule.h): reads
// "n_mats steps clusters group_bytes lag" (group_bytes < 0: the library's
// default order) then n_mats lines "rows cols" on stdin, builds the schedule
// and prints one line per item "mat mode k ti tj kt dep_target", then
// "makespan <simulated cycles>".
#include <cstdio>
#include <vector>

#include "schedule.h"

using namespace muonb200;

int main() {
  int n_mats = 0, steps = 0, clusters = 0, lag = 0;
  double group_bytes = 0.0;
  if (std::scanf("%d %d %d %lf %d", &n_mats, &steps, &clusters, &group_bytes, &lag) != 5)
    return 2;
  const SchedPolicy pol = group_bytes < 0 ? default_policy() : SchedPolicy{group_bytes, lag};
  std::vector<SchedMatrix> mats(n_mats);
  long long per_step = 0;
  for (int i = 0; i < n_mats; ++i) {
    int r = 0, c = 0;
    if (std::scanf("%d %d", &r, &c) != 2) return 2;
    SchedMatrix& s = mats[i];
    s.m = r < c ? r : c;
    s.n = r < c ? c : r;
    s.t2 = (s.m + 255) / 256;
    s.tn = (s.n + 255) / 256;
    per_step += s.t2 * (s.t2 + 1) + s.t2 * s.tn;
  }
  std::vector<SchedItem> out(per_step * steps);
  std::vector<SchedGroup> groups(static_cast<size_t>(n_mats) * steps * 3);
  std::vector<int> order(2 * static_cast<size_t>(n_mats) + 1);
  std::vector<double> cl(clusters);
  const long long n = build_schedule(mats.data(), n_mats, steps, clusters, pol, out.data(),
                                     static_cast<long long>(out.size()), groups.data(),
                                     order.data(), cl.data());
  if (n < 0) return 3;
  for (long long i = 0; i < n; ++i)
    std::printf("%d %d %d %d %d %d %d\n", out[i].mat, out[i].mode, out[i].k, out[i].ti,
                out[i].tj, out[i].kt, out[i].dep_target);
  // The device check (sched_item_valid) must accept every item of the list
  // and reject each of six corruptions of it.
  long long accepted = 0, missed = 0;
  for (long long i = 0; i < n; ++i) {
    const SchedItem& it = out[i];
    const SchedMatrix& mm = mats[it.mat];
    auto valid = [&](int mode, int k, int ti, int tj, int kt, int dep) {
      return sched_item_valid(mode, k, ti, tj, kt, dep, mm.m, mm.n, steps);
    };
    if (valid(it.mode, it.k, it.ti, it.tj, it.kt, it.dep_target)) ++accepted;
    const bool bad[6] = {
        valid(it.mode, it.k, it.ti + mm.t2, it.tj, it.kt, it.dep_target),
        valid(it.mode, it.k, it.ti, it.mode == kModeApply ? it.tj + mm.tn : it.tj + mm.t2,
              it.kt, it.dep_target),
        valid(it.mode, it.k, it.ti, it.tj, it.kt + 1, it.dep_target),
        valid(it.mode, steps, it.ti, it.tj, it.kt, it.dep_target),
        valid(3, it.k, it.ti, it.tj, it.kt, it.dep_target),
        valid(it.mode, it.k, it.ti, it.tj, it.kt, it.dep_target + 2)};
    for (bool b : bad) missed += b ? 1 : 0;
  }
  std::printf("checks %lld %lld\n", accepted, missed);
  double mk = 0;
  for (double t : cl) mk = t > mk ? t : mk;
  std::printf("makespan %.0f\n", mk);
  return 0;
}
