"""CPU check of the tensor-core kernel's share-out of the forward transform.

A block pair that no warp transforms leaves the issuer waiting on it until its
bounded wait runs out (the layer then fails); one that two warps transform
races.  The kernel's assignment functions (`pair_by_epilogue`, `pair_group`
and the constants they use) are taken verbatim from spectral_tc.cu, compiled
into a host program with nvcc, and run through the same loops the transform
and epilogue warps run, for every mode and every number of block pairs (1..10):
every block pair of a tile must be transformed by exactly one two-warp group.
"""

import os
import re
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "group_wise_dft_b200", "csrc")


def _roles_source():
    src = open(os.path.join(CSRC, "spectral_tc.cu")).read()
    consts = "\n".join(re.findall(r"^constexpr int k(?:NumDftWarps|NumEpiWarps|MaxFin|MaxBlocks|MaxPairs) = [^;]+;",
                                  src, flags=re.M))
    start = src.index("constexpr int kDftWarpsPerGroup")
    end = src.index("constexpr uint32_t kTmemCols")
    return consts + "\n" + src[start:end]


HARNESS = r"""
#include <cstdio>
#include "tc_pack_math.cuh"
namespace eqlin {
%s
}
using namespace eqlin;
template <int MODE>
int check() {
  int bad = 0;
  for (int nstage = 1; nstage <= kMaxPairs; ++nstage) {
    int count[kMaxPairs] = {};
    // transform groups, as the transform warps' loop
    for (int grp = 0; grp < kDftGroups; ++grp)
      for (int jp = grp; jp < nstage; ++jp) {
        if (pair_by_epilogue<MODE>(jp) || pair_group<MODE>(jp) != grp) continue;
        ++count[jp];
      }
    // epilogue help groups, as the epilogue warps' loop
    if (epilogue_helps<MODE>())
      for (int hgrp = 0; hgrp < kEpiHelpGroups; ++hgrp)
        for (int jp = kDftGroups + hgrp; jp < nstage && pair_by_epilogue<MODE>(jp); jp += kEpiHelpGroups)
          ++count[jp];
    for (int jp = 0; jp < nstage; ++jp)
      if (count[jp] != 1) { printf("mode %%d nstage %%d pair %%d: %%d groups\n", MODE, nstage, jp, count[jp]); ++bad; }
  }
  return bad;
}
int main() {
  int bad = check<kModeCyclic8>() + check<kModeD8>() + check<kModeNegacyclic8>() + check<kModeCyclic4>();
  // the accumulator-empty barrier counts every warp that arrives on it
  if (epilogue_warps<kModeD8>() != kNumEpiWarps + kD8HelpWarps) ++bad;
  if (epilogue_warps<kModeNegacyclic8>() != kNumEpiWarps + kD8HelpWarps) ++bad;
  // a mode whose epilogue warps help the transform must not also have
  // transform warps helping the epilogue
  if (epilogue_helps<kModeD8>() || epilogue_helps<kModeNegacyclic8>()) ++bad;
  if (epilogue_warps<kModeCyclic8>() != kNumEpiWarps) ++bad;
  if (kD8HelpWarps > kNumDftWarps || kD8HelpWarps %% 4 != 0) ++bad;   // whole lane quarters
  printf("bad %%d\n", bad);
  return bad != 0;
}
"""


@pytest.fixture(scope="module")
def harness(tmp_path_factory):
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(nvcc):
        pytest.skip("nvcc not available")
    d = tmp_path_factory.mktemp("roles")
    src = d / "roles.cu"
    src.write_text(HARNESS % _roles_source())
    exe = d / "roles"
    subprocess.run([nvcc, "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a", "-I", CSRC,
                    "-o", str(exe), str(src)], check=True, capture_output=True)
    return str(exe)


def test_every_block_pair_has_exactly_one_transforming_group(harness):
    out = subprocess.run([harness], capture_output=True, text=True)
    assert out.returncode == 0, out.stdout
    assert out.stdout.strip().endswith("bad 0")
