"""Host-side checks of libtq (no GPU needed): the library loads, exports every
entry point include/tq.h declares, rejects bad arguments, and its host tables
(an independent second implementation) agree with the oracle."""
import os
import re

import numpy as np
import pytest

import online_vector_quantization_b200 as tq
from oracle import tq_oracle as o

HEADER = os.path.join(os.path.dirname(os.path.dirname(__file__)), "include", "tq.h")


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(tq_[a-z0-9_]+)\s*\(", src)))


def test_every_declared_symbol_is_exported():
    names = declared_functions()
    assert len(names) >= 15
    for n in names:
        assert hasattr(tq._lib, n), n
        assert n in tq.EXPORTED, n


@pytest.mark.parametrize("d,b", [(128, 1), (128, 2), (128, 3), (128, 4), (64, 3), (256, 2), (128, 5), (64, 7),
                                 (128, 8)])
def test_codebook_matches_oracle(d, b):
    c, t = tq.tq_codebook(d, b)
    ref = o.lloyd_max(d, b)
    assert np.max(np.abs(c - ref.centroids)) < 1e-12
    assert np.max(np.abs(t - ref.bounds)) < 1e-12


@pytest.mark.parametrize("seed,d", [(0, 128), (12345, 128), (7, 16)])
def test_rotation_matches_oracle(seed, d):
    assert np.max(np.abs(tq.tq_rotation(seed, d) - o.rotation(seed, d))) < 1e-12


@pytest.mark.parametrize("seed,d", [(0, 128), (99, 128), (5, 8), (1, 512)])
def test_hadamard_rotation_matches_oracle(seed, d):
    assert np.array_equal(tq.tq_hadamard_rotation(seed, d), o.hadamard_rotation(seed, d))


def test_hadamard_rotation_rejects_non_power_of_two():
    with pytest.raises(tq.TqError) as e:
        tq.tq_hadamard_rotation(0, 96)
    assert e.value.status == 1


def test_qjl_matrix_matches_oracle():
    assert np.max(np.abs(tq.tq_qjl_matrix(3, 128, 128) - o.qjl_matrix(3, 128, 128))) < 1e-14


def test_host_argument_errors():
    with pytest.raises(tq.TqError) as e:
        tq.tq_codebook(2, 3)
    assert e.value.status == 1
    with pytest.raises(tq.TqError) as e:
        tq.Params(3, 3, d=64)
    assert e.value.status == 2
    with pytest.raises(tq.TqError) as e:
        tq.Params(5, 3)
    assert e.value.status == 2
    for bad in (dict(bits_k=6), dict(bits_k=8, mode_k=tq.TQ_MODE_PROD), dict(bits_k=8, mixed_k=1)):
        # 8-bit codes: MSE mode, uniform rows only
        args = dict(bits_k=3, bits_v=3)
        args.update(bad)
        with pytest.raises(tq.TqError) as e:
            tq.Params(args.pop("bits_k"), args.pop("bits_v"), **args)
        assert e.value.status == 2, bad
    with pytest.raises(tq.TqError) as e:
        tq.Params(3, 3, mixed_k=1, mode_k=tq.TQ_MODE_PROD)
    assert e.value.status == 2
    with pytest.raises(tq.TqError) as e:
        tq.Params(4, 4, mixed_k=1)
    assert e.value.status == 2
    with pytest.raises(tq.TqError) as e:
        tq.Params(3, 3, rotation=7)
    assert e.value.status == 1
    assert tq._lib.tq_cache_bytes(None, 1, 1, 64, 0) == 0
    assert tq._lib.tq_decode_workspace_bytes(None, 1, 8, 8, 128) == 0


def test_header_is_plain_c_and_links(tmp_path):
    """include/tq.h compiles as C99 with warnings as errors, and a C program
    links against libtq.so and calls a host entry point through it."""
    import shutil
    import subprocess

    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    lib_dir = os.path.dirname(tq.__file__)
    prog = tmp_path / "probe.c"
    prog.write_text(
        '#include "tq.h"\n#include <stdio.h>\n'
        "int main(void) {\n"
        "  double c[8], t[7];\n"
        "  if (tq_codebook(128, 3, c, t) != TQ_OK) return 1;\n"
        "  if (tq_codebook(2, 3, c, t) != TQ_ERR_ARG) return 2;\n"
        '  printf("%.12f\\n", c[7]);\n'
        "  return 0;\n}\n")
    exe = tmp_path / "probe"
    r = subprocess.run([cc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.dirname(HEADER), str(prog),
                        "-L", lib_dir, "-ltq", "-Wl,-rpath," + lib_dir, "-o", str(exe)],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, (r.returncode, r.stderr)
    assert abs(float(r.stdout) - o.lloyd_max(128, 3).centroids[7]) < 1e-12
