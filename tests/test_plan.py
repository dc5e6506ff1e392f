"""Host logic of the launch plan (protein_structure_models_b200/csrc/plan.h),
checked on the CPU: a small C++ harness includes plan.h, runs make_plan for the
workload shapes and edge cases, and prints the plan; the tests check the
resource limits the kernels rely on (shared memory, tensor-memory columns,
ring depth), the workspace layout (aligned, disjoint, in order), the fast
divisors against the quantities they divide by, and the mode choices."""
import json
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "protein_structure_models_b200", "csrc")

# B, N, H, D, Dv, P, Q, Cz, R, Cout, f32
CASES = {
    "w0": (1, 32, 4, 16, 16, 4, 8, 8, 2, 32, 1),
    "w1": (8, 256, 8, 16, 16, 4, 8, 128, 2, 256, 0),
    "w2": (1, 2048, 8, 32, 32, 8, 8, 64, 2, 256, 0),
    "w3-512": (1, 512, 8, 16, 16, 4, 8, 128, 2, 256, 0),
    "w3-4096": (1, 4096, 8, 16, 16, 4, 8, 128, 2, 256, 0),
    "w3-16384": (1, 16384, 8, 16, 16, 4, 8, 128, 2, 256, 0),
    "w4": (512, 150, 8, 16, 16, 4, 8, 64, 2, 256, 0),
    "n1": (2, 1, 3, 5, 3, 3, 5, 7, 3, 20, 0),
    "n300-f32": (2, 300, 3, 5, 3, 3, 5, 7, 3, 20, 1),
    "odd-cz": (1, 1000, 4, 8, 8, 2, 3, 5, 1, 17, 0),
    "too-long": (1, 140000, 2, 8, 8, 2, 2, 8, 1, 8, 0),
    "too-many-points": (1, 64, 2, 8, 8, 65, 2, 8, 1, 8, 0),
    "bad-dims": (1, 0, 2, 8, 8, 2, 2, 8, 1, 8, 0),
}

HARNESS = r"""
#include <cstdio>
#include <cstdlib>
#include "plan.h"
#include "bwd_plan.h"
using namespace fipa;
int main(int argc, char** argv) {
  int v[11];
  for (int i = 0; i < 11; ++i) v[i] = atoi(argv[1 + i]);
  Plan p; const char* why = "";
  int rc = make_plan(p, v[0], v[1], v[2], v[3], v[4], v[5], v[6], v[7], v[8], v[9], v[10], &why);
  printf("{\"rc\": %d, \"why\": \"%s\"", rc, why);
  if (rc == 0) {
    printf(", \"Kq\": %d, \"KHp\": %d, \"VHp\": %d, \"Zp\": %d, \"nKH\": %d, \"nZ\": %d, \"nQc\": %d, \"nqz\": %d",
           p.Kq, p.KHp, p.VHp, p.Zp, p.nKH, p.nZ, p.nQc, p.nqz);
    printf(", \"vbuf\": %d, \"nQres\": %d, \"nVB\": %d, \"nst\": %d, \"core_smem\": %zu, \"tmemO\": %d, \"Ocols\": %d",
           p.vbuf, p.nQres, p.nVB, p.nst, p.core_smem, p.tmemO, p.Ocols);
    printf(", \"Kg\": %d, \"Kgp\": %d, \"F\": %d, \"ntile_out\": %d, \"gemm_ks\": %d, \"gemm_nks\": %d, \"gemm_nst\": %d, \"gemm_smem\": %zu",
           p.Kg, p.Kgp, p.F, p.ntile_out, p.gemm_ks, p.gemm_nks, p.gemm_nst, p.gemm_smem);
    printf(", \"lift_res\": %d, \"lift_ctas\": %d, \"lift_smem\": %zu, \"nT\": %d, \"row0\": %d, \"row1\": %d",
           p.lift_res, p.lift_ctas, p.lift_smem, p.nT, p.row0, p.row1);
    printf(", \"fd\": {\"H\": [%u, %d], \"nK8\": [%u, %d], \"nZ8\": [%u, %d], \"nV8\": [%u, %d], \"Cz\": [%u, %d]}",
           p.fd_H.d, p.H, p.fd_nK8.d, p.KHp / 8, p.fd_nZ8.d, p.Zp / 8, p.fd_nV8.d, p.VHp / 8, p.fd_Cz.d, p.Cz);
    const size_t offs[] = {p.off_Q, p.off_KH, p.off_VH, p.off_Z, p.off_QP, p.off_KP, p.off_kvec, p.off_qvec,
                           p.off_orig, p.off_flag, p.off_stats, p.off_feat, p.off_wT, p.off_rowflag, p.total};
    printf(", \"offs\": [");
    for (int i = 0; i < 15; ++i) printf("%s%zu", i ? ", " : "", offs[i]);
    printf("]");
    BwdPlan b; const char* bwhy = "";
    const int brc = make_bwd_plan(b, p, &bwhy);
    printf(", \"bwd\": {\"rc\": %d, \"why\": \"%s\"", brc, bwhy);
    if (brc == 0) {
      printf(", \"q_smem\": %zu, \"k_smem\": %zu, \"q_nst\": %d, \"k_nst\": %d, \"nQr\": %d, \"nOc\": %d, \"k_nres\": %d",
             b.q_smem, b.k_smem, b.q_nst, b.k_nst, b.nQr, b.nOc, b.k_nres);
      printf(", \"tmDS\": %d, \"tmDQ\": %d, \"tmDK\": %d, \"tmDV\": %d, \"tmDZ\": %d, \"Vw\": %d, \"Kr\": %d, \"Kk\": %d, \"Fp\": %d",
             b.tmDS, b.tmDQ, b.tmDK, b.tmDV, b.tmDZ, b.Vw, b.Kr, b.Kk, b.Fp);
      const size_t bo[] = {b.off_lp, b.off_osave, b.off_dfeat, b.off_fhi, b.off_flo, b.off_duhi, b.off_dulo,
                           b.off_whi, b.off_wlo, b.off_dO, b.off_dvec, b.off_rloc, b.off_dz1u, b.off_qres, b.off_du,
                           b.off_kres, b.off_dz2h, b.off_dwpart, b.off_wbpart, b.off_gpart, b.total};
      printf(", \"offs\": [");
      for (int i = 0; i < 21; ++i) printf("%s%zu", i ? ", " : "", bo[i]);
      printf("]");
    }
    printf("}");
  }
  printf("}\n");
  return 0;
}
"""


@pytest.fixture(scope="module")
def plans(tmp_path_factory):
    if shutil.which("g++") is None:
        pytest.skip("g++ not available")
    d = tmp_path_factory.mktemp("plan")
    src, exe = d / "plan_harness.cpp", d / "plan_harness"
    src.write_text(HARNESS)
    inc = ["-I", CSRC, "-I", os.path.join(ROOT, "include")]
    cuda_inc = "/usr/local/cuda/include"
    if os.path.isdir(cuda_inc):
        inc += ["-I", cuda_inc]
    subprocess.run(["g++", "-std=c++17", "-O1", *inc, str(src), "-o", str(exe)], check=True)
    out = {}
    for name, dims in CASES.items():
        r = subprocess.run([str(exe), *map(str, dims)], check=True, capture_output=True, text=True)
        out[name] = json.loads(r.stdout)
    return out


def _ok(plans):
    return {k: v for k, v in plans.items() if v["rc"] == 0}


def test_supported_and_rejected_shapes(plans):
    for name in ("w0", "w1", "w2", "w3-512", "w3-4096", "w3-16384", "w4", "n1", "n300-f32", "odd-cz"):
        assert plans[name]["rc"] == 0, (name, plans[name]["why"])
    assert plans["too-long"]["rc"] == 2 and "131072" in plans["too-long"]["why"]
    assert plans["too-many-points"]["rc"] == 2
    assert plans["bad-dims"]["rc"] == 1


def test_core_fits_shared_and_tensor_memory(plans):
    for name, p in _ok(plans).items():
        assert p["core_smem"] <= 232448, name                   # 227 KB opt-in per block
        assert p["nst"] >= 3, name                              # ring depth the pipeline needs
        chunks = p["nQres"] + (p["nVB"] if p["vbuf"] else 0) + p["nst"]
        assert chunks * 16384 < p["core_smem"], name           # Qhat + value buffer + ring + tail
        assert p["tmemO"] + p["Ocols"] <= 512, name             # S, P and O in one CTA's columns
        assert p["gemm_smem"] <= 232448 and p["lift_smem"] <= 160 * 1024, name


def test_row_widths_are_whole_tma_chunks(plans):
    for name, p in _ok(plans).items():
        for key in ("Kq", "KHp", "VHp", "Zp", "Kgp"):
            assert p[key] % 64 == 0, (name, key)
        assert p["Kq"] == p["KHp"] + p["nqz"] * p["Zp"], name
        assert p["nQc"] * 64 == p["Kq"], name
        assert p["Kg"] <= p["Kgp"] < p["Kg"] + 64, name


def test_workspace_regions_are_aligned_disjoint_and_ordered(plans):
    for name, p in _ok(plans).items():
        offs = p["offs"]
        assert offs[0] == 0, name
        for a, b in zip(offs, offs[1:]):                        # the last entry is the total size
            assert a % 256 == 0 and a <= b, name


def test_fast_divisors_divide_by_what_they_claim(plans):
    for name, p in _ok(plans).items():
        for key, (d, want) in p["fd"].items():
            assert d == want, (name, key)


def test_mode_choices(plans):
    assert plans["w1"]["vbuf"] == 0                 # two key tiles: ring-only
    assert plans["w4"]["vbuf"] == 0
    assert plans["w3-4096"]["vbuf"] == 1            # from 8 key tiles: value buffer
    assert plans["w3-16384"]["vbuf"] == 1
    assert plans["w2"]["vbuf"] == 1
    assert plans["n300-f32"]["vbuf"] == 0 and plans["w0"]["vbuf"] == 0   # float32: never
    assert plans["w1"]["lift_res"] == 4 and plans["w4"]["lift_res"] == 8
    for name, p in _ok(plans).items():
        assert p["row0"] == 0 and p["row1"] == CASES[name][1], name   # full row range by default
        assert p["nT"] == (CASES[name][1] + 127) // 128, name
        assert p["lift_ctas"] == (CASES[name][1] + p["lift_res"] - 1) // p["lift_res"], name


def test_backward_plan_budgets_and_layout(plans):
    """The backward kernels' shared memory (<= 227 KB with the ring), tensor
    memory (S/dP + dS + dQhat, and S^T/dP^T + dK + dV + dz2, each <= 512
    columns) and the backward workspace regions (after the forward's,
    256-byte aligned, in order) for every supported bfloat16 shape; float32
    shapes are refused."""
    for name, p in _ok(plans).items():
        b = p["bwd"]
        if CASES[name][10] == 1:
            assert b["rc"] == 2 and "bfloat16" in b["why"], name
            continue
        assert b["rc"] == 0, (name, b["why"])
        assert b["q_smem"] <= 232448 and b["k_smem"] <= 232448, name
        assert b["q_nst"] >= 2 and b["k_nst"] >= 2, name
        assert b["tmDQ"] + 64 * b["nQr"] <= 512 and b["tmDS"] + 64 <= b["tmDQ"], name
        assert b["tmDZ"] + 64 * p["nZ"] <= 512 and b["tmDK"] >= 128, name
        assert b["Vw"] == 64 * b["nOc"] and b["nOc"] == p["VHp"] // 64 + p["nZ"], name   # dO = [head | pair]
        D, P, Dv, Q = CASES[name][3], CASES[name][5], CASES[name][4], CASES[name][6]
        assert b["Kr"] >= D + 3 * P + 5 and b["Kk"] >= D + 3 * P + 4 + Dv + 3 * Q, name
        assert b["Fp"] % 64 == 0 and b["Fp"] >= p["F"] + 1, name
        offs = b["offs"]
        assert offs[0] >= p["offs"][-1], name                  # after the forward's workspace
        for a, c in zip(offs, offs[1:]):
            assert a % 256 == 0 and a <= c, name
    # the protein-batch and length-sweep widths use every tensor-memory column on both sides
    b = plans["w3-16384"]["bwd"]
    assert b["tmDQ"] + 64 * b["nQr"] == 512 and b["tmDZ"] + 64 * plans["w3-16384"]["nZ"] == 512
