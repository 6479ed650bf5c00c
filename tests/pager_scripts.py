"""Runner of tests/golden/pager_scripts.txt (the page's own bookkeeping tests,
restated as operation scripts) against any pager with the interface of
oracle.pager.OraclePager: append(s, n) -> pos (raises on failure), popn(s, n),
reset(), num_free(), pages_used(s), seq_len(s), table()."""
from __future__ import annotations

import os
from collections import OrderedDict

HERE = os.path.dirname(os.path.abspath(__file__))


def load_scripts():
    cases = OrderedDict()
    with open(os.path.join(HERE, "golden", "pager_scripts.txt")) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            name, npg, ps, win, op, arg, ret, ln, used, free = [x.strip() for x in line.split(",")]
            cases.setdefault(name, {"setup": (int(npg), int(ps), int(win)), "ops": []})
            cases[name]["ops"].append((op, arg, ret, ln, used, free))
    return cases


def run_script(make_pager, num_pages_for, name, case, fail_exc):
    npg, ps, win = case["setup"]
    p = make_pager(npg, ps, [win] if win else [])
    for i, (op, arg, ret, ln, used, free) in enumerate(case["ops"]):
        where = f"{name} step {i} ({op} {arg})"
        if op == "pages":
            assert num_pages_for(int(arg), ps) == int(ret), where
            continue
        got = None
        if op == "grow":
            p.append(0, int(arg) - p.seq_len(0))
        elif op == "take":
            try:
                p.append(0, ps)
                got = str(p.table()[0][p.pages_used(0) - 1])
            except fail_exc:
                got = "x"
        elif op == "popn":
            got = str(p.popn(0, int(arg)))
        elif op == "reset":
            p.reset()
        else:
            raise ValueError(op)
        if ret != "-":
            assert got == ret, f"{where}: returned {got}, expected {ret}"
        if ln != "-":
            assert p.seq_len(0) == int(ln), f"{where}: length {p.seq_len(0)}"
        if used != "-":
            assert p.pages_used(0) == int(used), f"{where}: pages used {p.pages_used(0)}"
        if free != "-":
            assert p.num_free() == int(free), f"{where}: free {p.num_free()}"
