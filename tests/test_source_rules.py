"""Rules of the CUDA sources that no GPU test would catch reliably, checked on the text.

- No global load goes through the read-only path (`__ldg`, `ld.global.nc`): every kernel
  is a programmatic dependent launch whose lifetime overlaps its predecessor's, and that
  path requires data unchanged for the reading kernel's whole lifetime (a stale read
  shows only under unlucky timing).
- Every kernel that waits on its predecessor does so through pdl_wait_for(), which keeps
  the loads behind the wait; the bare pdl_wait() appears only where the code that follows
  launders its pointers itself.
- No copy uses cluster multicast.
"""
import glob
import os
import re

CSRC = os.path.join(os.path.dirname(__file__), "..", "scaling_aware_transpose_b200", "csrc")


def _code(path):
    """The file's text with // comments removed (string literals of inline PTX are kept)."""
    out = []
    for line in open(path):
        i = line.find("//")
        out.append(line if i < 0 else line[:i])
    return "".join(out)


def _sources():
    paths = sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh")) +
                   glob.glob(os.path.join(CSRC, "*.h")))
    assert paths, "no CUDA sources found"
    return paths


def test_no_read_only_path_loads():
    for p in _sources():
        code = _code(p)
        assert "__ldg(" not in code, f"{os.path.basename(p)} uses __ldg"
        assert not re.search(r"ld\.global\.nc|ld\.global\.[a-z0-9.]*\.nc", code), f"{os.path.basename(p)} uses ld.global.nc"


def test_waits_launder_their_pointers():
    bare = {}
    for p in _sources():
        if os.path.basename(p) == "common.cuh":
            continue  # defines both
        n = len(re.findall(r"\bpdl_wait\(\)", _code(p)))
        if n:
            bare[os.path.basename(p)] = n
    # gather_ids_kernel waits bare and then launders the one pointer it loads through
    assert bare == {"ep_dispatch.cu": 1}, bare
    assert "make_opaque(ids)" in _code(os.path.join(CSRC, "ep_dispatch.cu"))


def test_no_cluster_multicast():
    for p in _sources():
        assert "multicast::cluster" not in _code(p), f"{os.path.basename(p)} uses cluster multicast"
