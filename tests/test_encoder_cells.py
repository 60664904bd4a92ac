"""Exhaustive CPU check of the quantiser's NF4 encoder table.

The kernel finds a weight's code by a cell table (cell = rint(16 x + 16),
then the cell's base count plus one compare against the one threshold the
cell may hold).  This compiles that table, from the kernel's own constants
header, into a host program (encoder_cells_check.cpp) and compares the
table's code with the nearest of the oracle's 16 levels (binary64 distance,
ties to the lower code) for every binary32 x in [-1.0001, 1.0001]: the
normalised weights the encoder can see.  Each normalised weight is stored
as the index of the nearest of the 16 NF4 levels ("QLoRA",
learning-llms.pages.dev/topics/qlora, the sentence before the absmax
equation and the bullet on NF4); ties go to the lower code (a reading: the
pages do not say).
"""
import os
import shutil
import subprocess

import numpy as np
import pytest

from oracle import oracle as O

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(os.path.dirname(HERE), "bit_nf4_quantized_21_b200", "csrc")


@pytest.mark.skipif(shutil.which("g++") is None, reason="needs g++")
def test_cell_table_equals_nearest_level_for_every_binary32(tmp_path):
    exe = str(tmp_path / "encoder_cells_check")
    subprocess.run(["g++", "-O2", "-fopenmp", "-ffp-contract=off", "-std=c++17", "-I", CSRC,
                    "-o", exe, os.path.join(HERE, "encoder_cells_check.cpp")], check=True)
    levels = [float(v).hex() for v in np.asarray(O.nf4_levels(), np.float64)]
    r = subprocess.run([exe, *levels], capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout + r.stderr
    words = r.stdout.split()
    assert int(words[1]) == 2130708112   # every binary32 with |x| <= 1.0001
    assert int(words[3]) == 0
    assert int(words[5]) == 15           # a NaN (infinite-absmax block) reads the last cell
