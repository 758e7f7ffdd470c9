"""Plant plausible mistakes in a copy of the oracle and check that the pins catch
every one of them (CPU only; the planted copy lives in a temporary directory)."""
import os

import pytest

import oracle
import oracle_pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "ddt_oracle.c")

# (name, text to replace, replacement).  Each is a mistake a port could make.
MUTANTS = [
    ("drop rope term", "dot += bf16_to_double(qr[d]) * bf16_to_double(rrow[d]);", ";"),
    ("drop softmax scale", "s[j] = scale * dot;", "s[j] = dot;"),
    ("node does not see itself", "vis[(size_t)i * Q + i] = 1;", ";"),
    ("tree rows reversed", "vis_row[j - P]", "vis_row[T - 1 - j]"),
    ("lse without the max", "*lse = m + log(Z);", "*lse = log(Z);"),
    ("value from the wrong row", "const uint16_t* vrow = ckv + (int64_t)j * ckv_rs;",
     "const uint16_t* vrow = ckv + (int64_t)(j > 0 ? j - 1 : 0) * ckv_rs;"),
    ("mask bit order", "word |= (uint64_t)1 << k;", "word |= (uint64_t)1 << (63 - k);"),
    ("parents may point forward", "if (parents[i] < 0 || parents[i] >= i) ok = 0;",
     "if (parents[i] < 0 || parents[i] >= Q) ok = 0;"),
    ("last bit of each mask word dropped",
     "if (a < Q && vis[(size_t)i * Q + a]) word |= (uint64_t)1 << k;",
     "if (a < Q && k < 63 && vis[(size_t)i * Q + a]) word |= (uint64_t)1 << k;"),
    ("accept compares with the wrong target", "if (tok[c] == tgt[cur])", "if (tok[c] == tgt[c])"),
    ("accept skips the first child", "int c = first[cur];", "int c = first[cur] == -1 ? -1 : sib[first[cur]];"),
    ("walk limit one examination late", "if (examined > Q) {", "if (examined > Q + 1) {"),
    ("compaction writes one row late", "memcpy(ckv + (int64_t)(P + i) * ckv_rs",
     "memcpy(ckv + (int64_t)(P + i + (i + 1 < alen)) * ckv_rs"),
    ("compaction gathers in place (no staging)", ", s_ckv + (size_t)i * DL, sizeof(uint16_t) * DL);",
     ", ckv + (int64_t)(P + keep[i]) * ckv_rs, sizeof(uint16_t) * DL);"),
    ("depth off by one", "depth[i] = (i == 0) ? 0 : depth[parents[i]] + 1;",
     "depth[i] = (i == 0) ? 1 : depth[parents[i]] + 1;"),
    ("sibling weight keeps the node's own log-prob",
     "float w = x.logw - L[(size_t)(x.depth - 1) * K + x.rank];", "float w = x.logw;"),
    ("child weight from the node's own depth row", "float w = x.logw + L[(size_t)x.depth * K + 0];",
     "float w = x.logw + L[(size_t)(x.depth - 1) * K + 0];"),
    ("sibling weight from the parent's weight",
     "float w = x.logw - L[(size_t)(x.depth - 1) * K + x.rank];\n        w = w + L[(size_t)(x.depth - 1) * K + x.rank + 1];",
     "float w = lw[x.parent] + L[(size_t)(x.depth - 1) * K + x.rank + 1];"),
    ("only NaN log-probs rejected", "if (!isfinite(L[e])) st = ORC_BAD_LP;",
     "if (isnan(L[e])) st = ORC_BAD_LP;"),
    ("ties go to the latest insertion", "if (cand[c].logw > cand[best].logw) best = c;",
     "if (cand[c].logw >= cand[best].logw) best = c;"),
    ("token from rank 0", "ntk[node] = T[(size_t)(x.depth - 1) * K + x.rank];",
     "ntk[node] = T[(size_t)(x.depth - 1) * K];"),
    ("sibling hangs under the node", "cand[ncand++] = (orc_candidate){w, x.depth, x.rank + 1, x.parent};",
     "cand[ncand++] = (orc_candidate){w, x.depth, x.rank + 1, node};"),
    ("children stop one level early", "if (x.depth < D) {", "if (x.depth + 1 < D) {"),
]


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_mutant(tmp_path, name, old, new):
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor not found once: {old!r}"
    path = tmp_path / "mutant.c"
    path.write_text(src.replace(old, new))
    lib = oracle.compile_oracle(str(path), str(tmp_path / "libmutant.so"))
    orc = oracle.Oracle(lib)
    caught = []
    for pin in oracle_pins.ALL_PINS:
        try:
            pin(orc)
        except AssertionError:
            caught.append(pin.__name__)
    assert caught, f"no pin caught the planted mistake '{name}'"
