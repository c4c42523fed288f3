"""CPU checks of the measurement plumbing: the kernel-to-source map bench.py
uses for source digests names kernels that exist in those sources, every
committed ncu summary names a known kernel and a profile case bench.py can
run, and the summaries carry the fields bench.py reads (DRAM bytes per
launch and the source digest)."""
import glob
import os
import re

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "bitlinear_b1_fwd_b200", "csrc")


def _fields(path):
    kv = {}
    with open(path) as f:
        for line in f:
            if line.startswith("- ") and ":" in line:
                k, v = line[2:].split(":", 1)
                kv[k.strip()] = v.strip().strip("`")
    return kv


def test_kernel_source_map_names_real_kernels():
    for kernel, src in bench.KERNEL_SOURCE.items():
        with open(os.path.join(CSRC, src)) as f:
            text = f.read()
        assert re.search(r"\b%s\s*\(" % re.escape(kernel), text), f"{kernel} is not defined in {src}"


def test_every_kernel_of_the_library_is_mapped():
    defined = set()
    for path in glob.glob(os.path.join(CSRC, "*.cu")):
        with open(path) as f:
            text = f.read()
        # kernels are the functions declared right after __global__ (and
        # optional launch bounds or cluster dims)
        for m in re.finditer(r"__global__[^;{]*?\b(\w+_kernel)\s*\(", text):
            defined.add(m.group(1))
    assert defined, "no kernels found"
    assert defined <= set(bench.KERNEL_SOURCE), sorted(defined - set(bench.KERNEL_SOURCE))


def test_profiles_name_known_kernels_and_cases():
    paths = sorted(glob.glob(os.path.join(ROOT, "profiles", "ncu_*.md")))
    assert paths
    for p in paths:
        kv = _fields(p)
        assert kv.get("kernel") in bench.KERNEL_SOURCE, p
        assert kv.get("workload"), p
        assert re.fullmatch(r"[0-9a-f]{16}", kv.get("csrc_sha256", "")), p
        assert int(kv["dram_bytes_per_launch"]) > 0, p
        with open(p) as f:
            text = f.read()
        case = re.search(r"--profile-case (\w+)", text)
        assert case and case.group(1) in bench.PROFILE_CASES, p
        assert "--clock-control none" in text, p


def test_headline_roofline_kernels_have_profiles():
    """bench.py fills roofline.traffic from these two summaries when their
    digests match the sources."""
    names = {(_fields(p).get("kernel"), _fields(p).get("workload"))
             for p in glob.glob(os.path.join(ROOT, "profiles", "ncu_*.md"))}
    assert (bench.gemv_kernel_name(0, [(8640, 3200), (3200, 8640)]), "3b_decode") in names
    assert (bench.gemm_kernel_name(4096), "3b_prefill") in names


def test_every_kernel_has_an_ncu_summary():
    have = {_fields(p).get("kernel") for p in glob.glob(os.path.join(ROOT, "profiles", "ncu_*.md"))}
    assert set(bench.KERNEL_SOURCE) <= have, sorted(set(bench.KERNEL_SOURCE) - have)
