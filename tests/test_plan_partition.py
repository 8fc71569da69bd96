"""Host-side check of the fused kernel's launch plan and work split
(make_plan / build_task_list in fmoe_api.cu), built without a GPU.

For many shapes, grid sizes and the three modes the plan must fit shared
memory, respect every fixed-size per-block array the kernel indexes (router
rows and parts, unit and down-job counters, activation flags, stage words),
give every task a copy that fits one stage, and list the tasks in the order
the kernel relies on (router rows, then gate/up chunks, then the down jobs as
the last tasks).  Across the blocks of a grid every router row part, every
gate/up chunk and every down job must appear exactly once.  The benchmark
shapes must be plannable.  The program includes the API source with stub
launchers (nothing here reaches a kernel).
"""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "quantised_expert_ffn_router_b200", "csrc")

PROGRAM = r"""
#include "fmoe_api.cu"
#include <cstdio>
#include <map>
#include <tuple>

namespace fmoe {  // launchers are not exercised here
size_t batch_ws_bytes(int, int, int, int, int) { return 0; }
int batch_ws_carve(uint8_t*, int, int, int, int, int, BatchWs&) { return 1; }
int tc_encode_weight_map(const uint8_t*, int64_t, int, int, int, int, TmaDesc*) { return 1; }
int tc_encode_token_maps(const uint16_t*, int, int, TmaDesc*) { return 1; }
int launch_tc_gemm(int, bool, const TmaDesc&, const TmaDesc*, const TmaDesc*, const TcArgs&, int, void*) { return 1; }
int launch_batched(const BatchArgs&, const BatchWs&, int, void*) { return 1; }
int launch_topk_rows(const float*, int, int, int, int32_t*, float*, void*) { return 1; }
int launch_repack(const uint8_t*, uint8_t*, int, int, int, int, int, void*) { return 1; }
int launch_decode(const DecodePlan&, void*, bool, bool) { return 1; }
int launch_route_static(const uint16_t*, const float*, const uint16_t*, float, const uint16_t*, int, int, int, int,
                        int32_t*, float*, void*) { return 1; }
int launch_requant(const uint8_t*, uint8_t*, int, int, int, int, void*) { return 1; }
int route_static_prepare() { return 0; }
bool route_static_ready() { return true; }
int decode_max_smem_optin(int) { return 232448; }
int decode_occupancy(int, bool, int, int* b) { *b = 1; return 0; }
int zero_workspace(void*, size_t, void*) { return 1; }
}  // namespace fmoe

using namespace fmoe;
static int fails = 0, planned = 0;
#define CHECK(c, ...) do { if (!(c)) { printf("FAIL " __VA_ARGS__); printf("\n"); if (++fails > 20) return 1; } } while (0)

int check(int H, int E, int K, int I, int bits, int G, int mode, bool must_plan) {
  fmoe_config c = {};
  c.hidden = H; c.n_experts = E; c.top_k = K; c.inter = I; c.bits = bits; c.group = 64; c.n_layers = 1;
  c.max_tokens = 1; c.rms_eps = 1e-6f;
  DecodePlan P;
  const int max_smem = 232448;
  const bool ok = make_plan(c, G, mode, max_smem, P);
  CHECK(ok || !must_plan, "benchmark shape not plannable H%d E%d K%d I%d b%d G%d mode%d", H, E, K, I, bits, G, mode);
  if (!ok) return 0;
  ++planned;
  CHECK((int)P.smem_bytes <= max_smem, "smem %u", P.smem_bytes);
  CHECK(P.n_issuers >= 1 && P.n_issuers <= 32 && P.nstage % P.n_issuers == 0, "issuers %d nstage %d", P.n_issuers, P.nstage);
  CHECK(P.nstage + P.n_down_max <= 64, "stages %d + %d", P.nstage, P.n_down_max);
  CHECK(P.router_rows <= 16 && P.router_parts <= 4, "router rows %d parts %d", P.router_rows, P.router_parts);
  CHECK(P.units_per_cta <= 32 && P.rb_per_cta * P.n_slots <= 32 && 2 * P.n_slots <= 32, "per-block counters");
  CHECK(P.stage_bytes % 128 == 0 && P.off_ring % 128 == 0, "stage alignment");
  std::map<std::tuple<int, int, int>, int> seen;  // (type, item, chunk) -> count
  uint32_t list[kMaxTasks];
  for (int b = 0; b < G; ++b) {
    const int n = build_task_list(P, b, list);
    CHECK(n >= 0 && n <= kMaxTasks, "block %d has %d tasks", b, n);
    const int first_rb = G - 1 - b;
    const int my_rb = (P.n_slots > 0 && first_rb < P.n_rb) ? (P.n_rb - first_rb + G - 1) / G : 0;
    const int n_down = my_rb * P.n_slots * P.dn_chunks;
    CHECK(P.n_down_max == 0 || n_down <= P.n_down_max, "block %d: %d down jobs, %d stages", b, n_down, P.n_down_max);
    int phase = 0;
    for (int i = 0; i < n; ++i) {
      const uint32_t t = list[i], ty = task_type(t), idx = task_idx(t), slot = task_slot(t), ch = task_chunk(t);
      CHECK((int)ty >= phase, "block %d: task %d out of order", b, i);
      phase = (int)ty;
      CHECK((ty == kTaskDown) == (i >= n - n_down), "block %d: down jobs are not the last %d tasks", b, n_down);
      uint32_t bytes = 0;
      if (ty == kTaskRouter) {
        CHECK((int)idx < P.router_rows && (int)ch < P.router_parts, "router task");
        const int e = b + (int)idx * G;
        CHECK(e < E, "router row %d", e);
        bytes = (uint32_t)std::min(P.router_part_cols, H - (int)ch * P.router_part_cols) * 2;
        seen[{0, e, (int)ch}]++;
      } else if (ty == kTaskGateUp) {
        CHECK((int)idx < P.units_per_cta && (int)ch < P.gu_chunks && (int)slot < P.n_slots, "gate/up task");
        const int u = b + (int)idx * G;
        CHECK(u < P.total_units && u / P.units_per_slot == (int)slot, "unit %d slot %d", u, slot);
        bytes = (uint32_t)std::min(chunk_tiles(P.bits), P.gu_tiles - (int)ch * chunk_tiles(P.bits)) * P.tb;
        seen[{1, u, (int)ch}]++;
      } else {
        CHECK(ty == kTaskDown && (int)idx < P.rb_per_cta && (int)slot < P.n_slots && (int)ch < P.dn_chunks, "down task");
        const int rb = first_rb + (int)idx * G;
        CHECK(rb < P.n_rb, "row block %d", rb);
        bytes = (uint32_t)std::min(chunk_tiles(P.bits), P.dn_tiles - (int)ch * chunk_tiles(P.bits)) * P.tb;
        seen[{2, rb * 16 + (int)slot, (int)ch}]++;
      }
      CHECK(bytes > 0 && bytes <= P.stage_bytes && bytes % 16 == 0, "task bytes %u stage %u", bytes, P.stage_bytes);
    }
  }
  long want = 0;
  if (mode != kModeExpert) want += (long)E * P.router_parts;
  want += (long)P.total_units * P.gu_chunks + (long)P.n_rb * P.n_slots * P.dn_chunks;
  CHECK((long)seen.size() == want, "H%d E%d G%d mode%d: %zu distinct tasks, want %ld", H, E, G, mode, seen.size(), want);
  for (auto& kv : seen) CHECK(kv.second == 1, "a task is listed %d times", kv.second);
  return 0;
}

int main() {
  struct Shape { int H, E, K, I, bits; bool bench; };
  const Shape shapes[] = {{4096, 512, 4, 1024, 4, true}, {4096, 512, 4, 1024, 2, true}, {256, 16, 2, 128, 4, false},
                          {320, 37, 3, 192, 2, false},   {4096, 1000, 4, 1024, 4, false}, {256, 2048, 8, 128, 4, false},
                          {1024, 128, 8, 512, 4, false}, {64, 1, 1, 64, 4, false},        {4096, 64, 2, 4096, 4, false},
                          {2048, 300, 6, 768, 2, false}};
  for (const Shape& s : shapes)
    for (int G : {148, 132, 100, 37, 16})
      for (int mode : {kModeLayer, kModeExpert, kModeRoute})
        if (check(s.H, s.E, s.K, s.I, s.bits, G, mode, s.bench && G == 148)) return 1;
  if (fails) return 1;
  printf("planned %d OK\n", planned);
  return 0;
}
"""


def test_plan_fits_and_partitions_the_work(tmp_path):
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(nvcc):
        pytest.skip("nvcc not available")
    src = tmp_path / "plan_check.cu"
    src.write_text(PROGRAM)
    exe = tmp_path / "plan_check"
    out = subprocess.run([nvcc, "-std=c++17", "-O1", "-I", CSRC, "-o", str(exe), str(src)], capture_output=True,
                         text=True, timeout=600)
    assert out.returncode == 0, out.stderr[-3000:]
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=300)
    assert run.returncode == 0 and run.stdout.strip().endswith("OK"), run.stdout[-3000:] + run.stderr[-1000:]
    planned = int(run.stdout.split("planned")[1].split()[0])
    assert planned >= 100, planned  # most of the 150 (shape, grid, mode) cases have a plan
