"""Host logic of bench.py that decides what the JSON line may claim (CPU).

`ncu_traffic` reads a kernel's DRAM bytes per launch from a committed ncu
summary, and only while the kernel's source still has the hash recorded
beside the figure: counters taken on an older kernel must read as null.
"""
import hashlib
import os

import bench


def _profile(root, kernel, src_rel, digest, nbytes):
    os.makedirs(os.path.join(root, "profiles"), exist_ok=True)
    with open(os.path.join(root, "profiles", f"{kernel}_case.md"), "w") as f:
        f.write(f"# {kernel}\n\nsome table\n\n"
                f"traffic: kernel={kernel} source={src_rel} sha1={digest} bytes_per_launch={nbytes}\n")


def test_traffic_is_read_while_the_source_is_unchanged(tmp_path, monkeypatch):
    root = str(tmp_path)
    src_rel = "csrc/k.cu"
    os.makedirs(os.path.join(root, "csrc"))
    with open(os.path.join(root, src_rel), "wb") as f:
        f.write(b"__global__ void k() {}\n")
    digest = hashlib.sha1(open(os.path.join(root, src_rel), "rb").read()).hexdigest()
    _profile(root, "k_kernel", src_rel, digest, 5134448)
    monkeypatch.setattr(bench, "ROOT", root)
    got = bench.ncu_traffic("k_kernel")
    assert got == {"bytes_per_launch": 5134448, "profile": os.path.join("profiles", "k_kernel_case.md")}
    assert bench.ncu_traffic("other_kernel") is None


def test_traffic_is_null_once_the_source_changes(tmp_path, monkeypatch):
    root = str(tmp_path)
    src_rel = "csrc/k.cu"
    os.makedirs(os.path.join(root, "csrc"))
    path = os.path.join(root, src_rel)
    with open(path, "wb") as f:
        f.write(b"__global__ void k() {}\n")
    digest = hashlib.sha1(open(path, "rb").read()).hexdigest()
    _profile(root, "k_kernel", src_rel, digest, 123)
    with open(path, "ab") as f:   # even a comment is a different source
        f.write(b"// changed\n")
    monkeypatch.setattr(bench, "ROOT", root)
    assert bench.ncu_traffic("k_kernel") is None
    os.remove(path)
    assert bench.ncu_traffic("k_kernel") is None


def test_committed_summaries_name_their_commands_and_kernels():
    # every committed summary that carries a traffic line names a source file
    # that exists, and gives the ncu command it came from
    import glob
    import re

    pat = re.compile(r"traffic: kernel=(\S+) source=(\S+) sha1=([0-9a-f]{40}) bytes_per_launch=(\d+)")
    found = 0
    for path in glob.glob(os.path.join(bench.ROOT, "profiles", "*.md")):
        text = open(path).read()
        assert "ncu " in text and "--clock-control none" in text, path
        for m in pat.finditer(text):
            found += 1
            assert os.path.exists(os.path.join(bench.ROOT, m.group(2))), m.group(2)
            assert int(m.group(4)) > 0
    assert found >= 2


def test_job_throughput_counts_every_rank():
    # whole-job GB/s: every rank streams its bytes in the slowest rank's time
    assert bench.job_gbs(1, 1e9, 1000.0) == 1.0
    assert bench.job_gbs(4, 1e9, 1000.0) == 4.0
