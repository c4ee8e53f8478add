"""Regression pin: the oracle still produces the stored container fixture.

The fixture (tests/golden/oracle_containers.txt) was written by
tests/golden/make_golden.py from the oracle alone; a mismatch means the
format changed and the change must cite the passage or reading behind it.
"""
import os

import numpy as np

from oracle import oracle as o

FIX = os.path.join(os.path.dirname(__file__), "golden", "oracle_containers.txt")


def test_oracle_reproduces_fixture():
    tab = o.Tables(2, sign_seed=0)
    streams = {"K": tab.k, "V": tab.v}
    seen = 0
    with open(FIX) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            parts = line.split()
            if parts[0] == "table":
                st = streams[parts[1]]
                vals = parts[3:]
                if parts[2] == "freq":
                    assert [int(v) for v in vals] == [int(v) for v in st.freq]
                else:
                    arr = {"yf_bits": st.yf, "tf_bits": st.tf, "cost_bits": st.cost}[parts[2]]
                    assert ["%08x" % v for v in arr.view(np.uint32)] == vals
            elif parts[0] == "signs":
                assert [int(v) for v in parts[1:]] == [int(v) for v in tab.signs.reshape(-1)]
            elif parts[0] == "vec":
                st = streams[parts[1]]
                head = int(parts[3])
                body = line.split(" ", 4)[4]
                xs, ss, hexs = [p.strip() for p in body.split("|")]
                x = np.array([int(w, 16) for w in xs.split()], dtype=np.uint32).view(np.float32)
                cont, syms, _, bad = o.encode_vectors(st, tab.signs, x[None], np.array([head], np.int32))
                assert bad == 0
                assert [int(v) for v in ss.split()] == [int(v) for v in syms[0]]
                assert cont[0].tobytes().hex() == hexs
                seen += 1
    assert seen == 12
