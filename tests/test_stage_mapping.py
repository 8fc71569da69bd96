"""Host-side check of the ring mapping the fused kernel's producer and
consumers both compute (task_stage_of in fmoe_internal.h), across layers of
a multi-layer launch.

The producer's lane i % n_issuers issues ring task i of every layer; the
consumers wait for a stage's phase by parity, which is only unambiguous if
every stage is refilled in order, by one lane, with fills 0, 1, 2, ... and
no two tasks of a layer share a (stage, fill).  A small host program (built
with nvcc, no GPU needed) walks the issue order of many plan shapes for
several layers and checks exactly that.  It also checks that down jobs keep
their own stages (fill = layer), that layer 0 maps like a single-layer launch,
and that the per-lane counters the producer keeps (ring_advance) give the same
positions at every issue.
"""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "quantised_expert_ffn_router_b200", "csrc")

PROGRAM = r"""
#include <cstdio>
#include <vector>
#include "fmoe_internal.h"
using namespace fmoe;

int main() {
  long checked = 0;
  for (int ni = 1; ni <= 8; ++ni)
    for (int per = 1; per <= 6; ++per) {
      const int nstage = ni * per;
      for (int n_tasks = 1; n_tasks <= 96; ++n_tasks)
        for (int n_down = 0; n_down < n_tasks && n_down <= 32; n_down += (n_down < 12 ? 1 : 5)) {
          const int ring_end = n_tasks - n_down, n_layers = 5;
          std::vector<int> next_fill(nstage + n_down, 0), owner(nstage + n_down, -1);
          // the producer's per-lane counters (ring_advance), one pair per lane
          std::vector<int> lane_slot(ni, 0), lane_fill(ni, 0);
          for (int l = 0; l < n_layers; ++l) {
            // issue order: rounds of ni consecutive tasks, lanes in parallel;
            // per lane the order is its tasks in increasing index
            for (int lane = 0; lane < ni; ++lane)
              for (int i = lane; i < ring_end; i += ni) {
                int s, f;
                task_stage_of(nstage, ni, n_tasks, n_down, i, s, f, l);
                if (lane_slot[lane] * ni + lane != s || lane_fill[lane] != f) {
                  printf("FAIL counters disagree ni=%d nstage=%d tasks=%d down=%d l=%d i=%d\n", ni, nstage, n_tasks,
                         n_down, l, i);
                  return 1;
                }
                ring_advance(per, lane_slot[lane], lane_fill[lane]);
                if (s < 0 || s >= nstage || s % ni != lane) {
                  printf("FAIL stage range/owner ni=%d nstage=%d tasks=%d down=%d l=%d i=%d s=%d\n", ni, nstage,
                         n_tasks, n_down, l, i, s);
                  return 1;
                }
                if (owner[s] >= 0 && owner[s] != lane) {
                  printf("FAIL two lanes fill stage %d\n", s);
                  return 1;
                }
                owner[s] = lane;
                if (f != next_fill[s]) {
                  printf("FAIL fill order ni=%d nstage=%d tasks=%d down=%d l=%d i=%d s=%d fill=%d want=%d\n", ni,
                         nstage, n_tasks, n_down, l, i, s, f, next_fill[s]);
                  return 1;
                }
                ++next_fill[s];
                if (l == 0) {
                  int s0, f0;
                  task_stage(nstage, ni, i, s0, f0);
                  if (s0 != s || f0 != f) {
                    printf("FAIL layer 0 differs from the single-layer mapping at i=%d\n", i);
                    return 1;
                  }
                }
                ++checked;
              }
            for (int i = ring_end; i < n_tasks; ++i) {
              int s, f;
              task_stage_of(nstage, ni, n_tasks, n_down, i, s, f, l);
              if (s != nstage + (i - ring_end) || f != l || f != next_fill[s]) {
                printf("FAIL down stage i=%d l=%d s=%d f=%d\n", i, l, s, f);
                return 1;
              }
              ++next_fill[s];
              ++checked;
            }
          }
        }
    }
  printf("OK %ld\n", checked);
  return 0;
}
"""


def test_ring_mapping_refills_in_order(tmp_path):
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(nvcc):
        pytest.skip("nvcc not available")
    src = tmp_path / "stage_map.cu"
    src.write_text(PROGRAM)
    exe = tmp_path / "stage_map"
    subprocess.run([nvcc, "-std=c++17", "-O1", "-I", CSRC, "-o", str(exe), str(src)], check=True,
                   capture_output=True, timeout=300)
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=300)
    assert out.returncode == 0 and out.stdout.startswith("OK"), out.stdout + out.stderr
