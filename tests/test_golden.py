"""Values the pages print, checked against this repository's byte accounting.

The memory table of "Evoformer: the memory wall ZeRO cannot move" (section
"Where the memory goes") gives the pair representation and the triangle
attention logits at c_z = 128, 4 heads, bf16.  The same N^3 * H * bytes
formula sizes the tensor this library never materialises, and the memory test
on the GPU uses it as the bar that peak memory must stay far below.
"""
import os

import pytest

from evoformer_pair_bias_b200.workloads import WORKLOADS, logits_bytes, pair_rep_bytes

HERE = os.path.dirname(os.path.abspath(__file__))


def _rows():
    with open(os.path.join(HERE, "golden", "triangle_logits_memory.tsv")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            n, pr, lg, ratio = line.split()
            yield int(n), float(pr), float(lg), float(ratio)


@pytest.mark.parametrize("n,pair_mb,logit_mb,ratio", list(_rows()))
def test_memory_table(n, pair_mb, logit_mb, ratio):
    assert round(pair_rep_bytes(n, 128, 2) / 1e6, 1) == pair_mb
    assert round(logits_bytes(n, 4, 2) / 1e6, 1) == logit_mb
    assert round(logits_bytes(n, 4, 2) / pair_rep_bytes(n, 128, 2), 1) == ratio


def test_long_case_fp32_logits_would_be_58_gb():
    w = WORKLOADS["tri_long_1536"]
    # one layer's logits over all rows: N_rows * H * N * N fp32
    assert round(w.logits * 4 / 1e9, 2) == 57.98
