"""The forward-backward kernel's shared-memory carve-up (fb_smem_layout in
csrc/bcjr_internal.h) for every team shape the bitshift launches can take,
with the host's staging decision (fb_xstage): regions are disjoint except
where sharing is intended, aligned for their vector and bulk-copy accesses,
and the staging never pushes a shape past the 227 KiB a CTA can have.
Host logic only: a small C++ program (tests/smem_layout_dump.cpp) prints
the layouts; no GPU is needed."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
MAX_SMEM = 227 * 1024  # opt-in dynamic shared memory per CTA on sm_100
FIELDS = ("L k adj alias nseq cluster NT tpc GL NV xs exA exF exB exBt mbar per_seq per_team red "
          "stage stageF stageK xst xstF cf total").split()


def _cuda_include():
    for d in (os.environ.get("CUDA_HOME", ""), "/usr/local/cuda"):
        if d and os.path.exists(os.path.join(d, "include", "cuda_runtime.h")):
            return os.path.join(d, "include")
    return None


@pytest.fixture(scope="module")
def layouts(tmp_path_factory):
    gxx, inc = shutil.which("g++"), _cuda_include()
    if not gxx or not inc:
        pytest.skip("needs g++ and the CUDA headers")
    exe = str(tmp_path_factory.mktemp("sld") / "sld")
    subprocess.run([gxx, "-std=c++17", "-O1", "-I", os.path.join(ROOT, "include"), "-I",
                    os.path.join(ROOT, "differentiable_bcjr_b200", "csrc"), "-I", inc,
                    os.path.join(ROOT, "tests", "smem_layout_dump.cpp"), "-o", exe], check=True)
    out = subprocess.run([exe], check=True, capture_output=True, text=True).stdout
    rows = [dict(zip(FIELDS, map(int, line.split()))) for line in out.splitlines()]
    assert len(rows) > 100
    return rows


def _regions(r):
    """(name, start, size) of every region in bytes, CTA-relative."""
    GL, NT, NV, nseq = r["GL"], r["NT"], r["NV"], r["nseq"]
    adj, alias = r["adj"], r["alias"]
    stg = nseq * NT if alias else 0
    reg = []
    for team in range(r["tpc"]):
        for x in range(nseq):
            b = team * r["per_team"] + x * r["per_seq"]
            reg.append((f"exA{team}.{x}", b + r["exA"], 2 * GL * 8))
            if adj:
                reg.append((f"exF{team}.{x}", b + r["exF"], 2 * GL * 4))
            if not alias:
                reg.append((f"exB{team}.{x}", b + r["exB"], 2 * GL * 8))
                if adj:
                    reg.append((f"exBt{team}.{x}", b + r["exBt"], 2 * GL * 4))
            reg.append((f"mbar{team}.{x}", b + r["mbar"], 32))
    reg.append(("red", r["red"], 4 * 128 * 4))
    reg.append(("stage", r["stage"], stg * NV * 4))
    if adj:
        reg.append(("stageF", r["stageF"], stg * NV * 4))
    reg.append(("stageK", r["stageK"], stg * 4))
    if r["xs"]:
        reg.append(("xst", r["xst"], nseq * 2 * GL * 8))
        if adj:
            reg.append(("xstF", r["xstF"], nseq * 2 * GL * 4))
    reg.append(("cf", r["cf"], NT * 16 * 4))
    return [x for x in reg if x[2] > 0]


def test_regions_are_disjoint_and_inside(layouts):
    for r in layouts:
        reg = _regions(r)
        for name, start, size in reg:
            assert 0 <= start and start + size <= r["total"], (r, name)
        for i, (n1, s1, z1) in enumerate(reg):
            for n2, s2, z2 in reg[i + 1:]:
                if s1 < s2 + z2 and s2 < s1 + z1:
                    # the adjoint's outgoing staging (forward sweep) shares room with
                    # the checkpoint staging (backward sweep)
                    shared = r["adj"] and {n1.rstrip("F"), n2.rstrip("F")} <= {"stage", "xst", "stageK"} \
                        and (n1.startswith("xst") != n2.startswith("xst"))
                    assert shared, (r, n1, n2)


def test_alignment(layouts):
    # 16 bytes: two-double / four-float stores into exA and exF, 16-byte
    # cp.async into the checkpoint staging, bulk copies out of xst / xstF (and
    # team and sequence bases, which every offset is relative to); 8 bytes:
    # the backward sweep's single-double and float-pair stores, mbarriers,
    # the float2 codeword pairs.
    for r in layouts:
        need = {"exA": 16, "exF": 16, "per_seq": 16, "per_team": 16, "stage": 16, "xst": 16, "exB": 8,
                "exBt": 8, "mbar": 8, "cf": 8}
        if r["adj"]:
            need.update(stageF=16, xstF=16)
        for f, a in need.items():
            assert r[f] % a == 0, (r, f)


def test_staging_rule_and_fit(layouts):
    for r in layouts:
        expect = r["cluster"] > 1 and r["k"] <= 2 and r["nseq"] <= 2 and (not r["adj"] or r["alias"])
        assert bool(r["xs"]) == expect, r
        if r["xs"]:
            assert r["total"] <= MAX_SMEM, r
    # the projection workload's launches (S = 2^16, k = 2, C = 1) stage and fit
    proj = [r for r in layouts if (r["L"], r["k"], r["alias"], r["nseq"]) == (16, 2, 1, 2)]
    assert len(proj) == 2 and all(r["xs"] and r["total"] <= MAX_SMEM and r["cluster"] == 8 for r in proj)
