"""The host pipeline's chunk schedule (no GPU): csrc/tara_host.cpp is compiled with g++ into a
small program (its two library-internal callees stubbed, never reached) that prints the chunk
sizes for many (planes, chunk cap) pairs; the sizes must cover every plane once, respect the
cap, ramp 1, 2, 4, ... up at the start and mirror it at the end, and split the middle evenly."""
import os
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "video_diffusion_attention_b200", "csrc")
CUDA = os.environ.get("CUDA_HOME", "/usr/local/cuda")

PROGRAM = r"""
#include <cstdio>
#include "tara_host.cpp"

namespace tara {
size_t forward_workspace_bytes(const tara_tensor*, const tara_token_meta*, const tara_params*) {
  return 0;
}
int forward_with_workspace(const tara_tensor*, const tara_tensor*, const tara_tensor*,
                           const tara_token_meta*, const tara_params*, tara_tensor*, float*,
                           void*, size_t, void*, long long) {
  return TARA_ERR_CUDA;
}
}  // namespace tara
extern "C" int tara_set_kernel_events(void*, void*) { return TARA_OK; }

int main() {
  const long long Ps[] = {1, 2, 3, 5, 8, 9, 10, 16, 17, 56, 100, 112, 1000};
  const long long Gs[] = {1, 2, 3, 4, 8, 9, 16, 121};
  for (long long P : Ps)
    for (long long G0 : Gs) {
      const long long G = G0 > P ? P : G0;   // the caller caps G at P
      std::printf("%lld %lld :", P, G);
      for (long long g : chunk_sizes(P, G)) std::printf(" %lld", g);
      std::printf("\n");
    }
  return 0;
}
"""


@pytest.fixture(scope="module")
def schedules(tmp_path_factory):
    d = tmp_path_factory.mktemp("chunks")
    src, exe = d / "chunks.cpp", d / "chunks"
    src.write_text(PROGRAM)
    lib = os.path.join(CUDA, "lib64")
    subprocess.check_call(["g++", "-std=c++17", "-O1", "-I", os.path.join(ROOT, "include"),
                           "-I", CSRC, "-I", os.path.join(CUDA, "include"), str(src),
                           "-o", str(exe), "-L", lib, "-lcudart", "-Wl,-rpath," + lib])
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60, check=True).stdout
    res = {}
    for line in out.strip().splitlines():
        head, sizes = line.split(":")
        P, G = (int(x) for x in head.split())
        res[(P, G)] = [int(x) for x in sizes.split()]
    return res


def test_every_plane_once_within_the_cap(schedules):
    assert len(schedules) > 50
    for (P, G), sizes in schedules.items():
        assert sum(sizes) == P, (P, G, sizes)
        assert all(1 <= g <= G for g in sizes), (P, G, sizes)


def test_ramp_up_and_down(schedules):
    for (P, G), sizes in schedules.items():
        head = []
        s, hs = 1, 0
        while s < G and 2 * (hs + s) <= P:
            head.append(s)
            hs += s
            s *= 2
        assert sizes[:len(head)] == head, (P, G, sizes)
        assert sizes[len(sizes) - len(head):] == head[::-1], (P, G, sizes)
        mid = sizes[len(head):len(sizes) - len(head)]
        if mid:
            assert max(mid) - min(mid) <= 1, (P, G, sizes)
            assert len(mid) == -(-(P - 2 * hs) // G), (P, G, sizes)


def test_headline_shot_schedule(schedules):
    # 56 heads of 27.4 MB planes, 9 planes per 1 GiB chunk
    assert schedules[(56, 9)] == [1, 2, 4, 8, 9, 9, 8, 8, 4, 2, 1]
    assert schedules[(8, 8)] == [1, 2, 2, 2, 1]
    assert schedules[(1, 1)] == [1]
