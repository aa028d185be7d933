"""The benchmarked kernel instances keep their working set in registers.

Compiles the hot-path sources with `ptxas -v` (the resource report the
compiler prints; nothing is disassembled) and checks the stack frame of each
benchmarked instance. A register array that the compiler can only address
with a run-time index is moved to local memory for the whole kernel; that
happened to the per-block code registers of the tensor-core encode (an
'if (b == e / JC) fld[b] = ...' patch inside a loop over flagged values)
and cost it 8 %. CPU only (nvcc cross-compiles); skipped without nvcc.
"""

import os
import re
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "kv_cache_vector_turboquant_b200", "csrc")


def _nvcc():
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    return None


_CACHE = {}


def _frames(source, tmp_path):
    """{mangled function name: (stack frame bytes, spill store bytes, spill load bytes)}
    (one compile per source file per session)"""
    if source in _CACHE:
        return _CACHE[source]
    nvcc = _nvcc()
    if nvcc is None:
        pytest.skip("nvcc not available")
    out = subprocess.run([nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-std=c++17", "-O3", "-Xptxas", "-v",
                          "-I" + os.path.join(ROOT, "include"), "-I" + CSRC, "-c", os.path.join(CSRC, source),
                          "-o", str(tmp_path / (source + ".o"))], capture_output=True, text=True)
    assert out.returncode == 0, out.stderr[-2000:]
    frames, current = {}, None
    for ln in out.stderr.splitlines():
        m = re.search(r"Function properties for (\S+)", ln)
        if m:
            current = m.group(1)
            continue
        m = re.search(r"(\d+) bytes stack frame, (\d+) bytes spill stores, (\d+) bytes spill loads", ln)
        if m and current is not None:
            frames[current] = tuple(int(v) for v in m.groups())
            current = None
    _CACHE[source] = frames
    return frames


def _instance(frames, pattern):
    hits = [v for k, v in frames.items() if re.search(pattern, k)]
    assert len(hits) == 1, (pattern, sorted(frames))
    return hits[0]


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_tensor_core_encode_has_no_stack_frame(tmp_path_factory, bits):
    frames = _frames("tq_encode_tc.cu", tmp_path_factory.mktemp("enc_tc"))
    assert _instance(frames, rf"encode_tc_kernelILi128ELi{bits}E") == (0, 0, 0)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("bits", [2, 3, 4])
def test_tensor_core_decode_frames(tmp_path_factory, d, bits):
    """The plain decode instances (Lb0: not the offset variant) have no stack
    frame; the offset-variant instances, at the 96-register cap of 18 warps
    with two more live values, are allowed a few bytes of spill."""
    frames = _frames("tq_decode_tc.cu", tmp_path_factory.mktemp("dec_tc"))
    assert _instance(frames, rf"decode_tc_kernelILi{d}ELi{bits}ELb0E") == (0, 0, 0)
    fb, st, ld = _instance(frames, rf"decode_tc_kernelILi{d}ELi{bits}ELb1E")
    assert fb <= 32 and st <= 32 and ld <= 64


def test_fused_attention_has_no_stack_frame(tmp_path_factory):
    frames = _frames("tq_attend_fast.cu", tmp_path_factory.mktemp("att"))
    assert _instance(frames, r"attend_fast_kernelILi128ELi8E") == (0, 0, 0)


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_cuda_core_encode_has_no_stack_frame(tmp_path_factory, bits):
    frames = _frames("tq_encode.cu", tmp_path_factory.mktemp("enc"))
    hits = [v for k, v in frames.items() if re.search(rf"encode_kernelILi128ELi{bits}E", k)]
    assert hits and all(v == (0, 0, 0) for v in hits), hits
