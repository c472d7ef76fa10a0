"""The dispatch-table parser on malformed files (CPU, no GPU needed): random
lines of plausible and implausible tokens, over-long lines, huge and negative
numbers, stray bytes.  Every file is either accepted or refused with
LQ_ERR_TABLE; nothing crashes, and a refused file leaves the table in force
unchanged.  (A table entry is checked again before every launch it selects,
so an accepted entry can never launch an invalid variant.)"""

import random

from quantized_linear_gemm_b200 import lq

TABLE = 7
TOKENS = ["fp8_dynamic", "w8a8_int8", "block_fp8", "block_fp8_ue8m0", "bogus", "#", "-1", "0", "1", "2", "3",
          "16", "24", "32", "128", "256", "4096", "99999999999999999999", "-99999999999999999999", "1e9", "0x10",
          "nan", "", "\t", "é", "\x00", "\x7f"]


def test_malformed_tables_are_refused_cleanly(tmp_path):
    rng = random.Random(0)
    base = lq.dispatch_table_size()
    accepted = refused = 0
    p = tmp_path / "t.txt"
    try:
        for _ in range(1500):
            lines = [" ".join(rng.choice(TOKENS) for _ in range(rng.randint(0, 14)))
                     for _ in range(rng.randint(0, 6))]
            if rng.random() < 0.1:
                lines.append("x" * rng.randint(1, 100000))
            p.write_text("\n".join(lines), encoding="utf-8")
            before = lq.dispatch_table_size()
            try:
                lq.load_dispatch_table(str(p))
                accepted += 1
            except lq.LQError as e:
                assert e.code == TABLE
                assert lq.dispatch_table_size() == before
                refused += 1
    finally:
        lq.load_dispatch_table(None)
    assert lq.dispatch_table_size() == base
    assert accepted > 0 and refused > 0
