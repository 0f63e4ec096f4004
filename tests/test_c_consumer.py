"""The C ABI used from C: a plain C program (tests/c/abi_host_check.c)
includes include/vark.h, links the in-tree libvark.so with gcc and runs the
host-side calls; its schedule, S-CAS finalisation and cache accounting must
equal the oracle's, and a device call on a host without a GPU must come back
as a status, not a crash."""
import os
import shutil
import subprocess

import numpy as np
import pytest

import kv_cache_compression_cas_b200 as vark
import oracle
from synth import SIDES_1024, SIDES_TINY

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def exe(tmp_path_factory):
    if shutil.which("gcc") is None:
        pytest.skip("no C compiler")
    lib = vark.LIB_PATH
    out = str(tmp_path_factory.mktemp("c") / "abi_host_check")
    subprocess.run(["gcc", "-std=c11", "-O1", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                    os.path.join(ROOT, "tests", "c", "abi_host_check.c"), lib, "-o", out,
                    f"-Wl,-rpath,{os.path.dirname(lib)}"], check=True, capture_output=True, text=True)
    return out


def _no_device():
    import torch
    return not torch.cuda.is_available()


def _run(exe, scas, sides, n_sinks, budget):
    L, H, S = scas.shape
    text = f"{L} {H} {S} {n_sinks} {budget}\n" + " ".join(map(str, sides)) + "\n" + \
           " ".join(repr(float(x)) for x in scas.ravel()) + "\n"
    # the device call uses placeholder host pointers: only where no GPU could run it
    args = [exe, "device"] if _no_device() else [exe]
    r = subprocess.run(args, input=text, capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, r.stderr
    return {ln.split()[0]: ln.split()[1:] for ln in r.stdout.strip().splitlines()}


@pytest.mark.parametrize("sides,L,H,budget", [(SIDES_TINY, 2, 3, 4000), (SIDES_1024, 4, 16, 1000)])
def test_c_program_matches_oracle(exe, sides, L, H, budget):
    S = len(sides)
    scas = np.round(np.random.default_rng(L * H).uniform(size=(L, H, S)), 4)
    out = _run(exe, scas, sides, 2, budget)
    assert int(out["version"][0]) == vark.vark_version()
    assert out["schedule"][0] == "0"
    keep = np.array(list(map(int, out["schedule"][1:])), dtype=np.uint8).reshape(L, H, S)
    ref = oracle.build_schedule(scas, sides, budget, 2)
    assert np.array_equal(keep, ref)
    assert out["finalize"][0] == "0"
    fin = np.array(list(map(float, out["finalize"][1:]))).reshape(L, H, S)
    mass = np.zeros((L, H, S, S))
    mass[:, :, :, S - 1] = scas.astype(np.float32)
    np.testing.assert_allclose(fin, oracle.scas_from_mass(mass, 1), rtol=1e-15, atol=0)
    assert out["cache"][0] == "0"
    cache = np.array(list(map(int, out["cache"][1:]))).reshape(S, L)
    assert np.array_equal(cache, oracle.cache_size_after_layer(ref, sides, 2, 64))
    # argument errors of device calls come back before any device work, from C too
    assert out["args"] == ["-1", "-2", "-3"]
    # no GPU here: a device call reports a status from the library's own table
    if _no_device():
        status = int(out["device"][0])
        assert status == -7 and out["device"][1].startswith("VARK")


def test_c_program_reports_infeasible_budget(exe):
    scas = np.full((1, 2, len(SIDES_TINY)), 0.5)
    out = _run(exe, scas, SIDES_TINY, len(SIDES_TINY), 100)   # every scale a sink, 1% budget
    assert out["schedule"] == ["-4"]
