"""The launch plan of the factorisation's corrections, checked on the CPU for
sizes the GPU tests do not reach.

The blocked Cholesky applies panel q's correction to every later block
column cb (and, for M^{-1}, row block cb): cb = q + 1 inside panel q + 1's
own kernel (look-ahead), every cb >= q + 2 through the side-stream products
(narrow, band and far, section comments in prepare.cu).  This test restates
the stream and event sequence the host code enqueues (one function below,
kept in step with enqueue_prepare) and checks three properties for every size:

  * coverage: each (q, cb >= q + 2) contribution is applied by exactly one
    product, for A (block columns) and for M^{-1} (row blocks);
  * the chain: every product writing block column / row block cb precedes
    panel cb in the launch graph (stream order plus event waits);
  * determinism: any two products that write the same block column (or row
    block) are ordered in the launch graph, so the additions into it happen
    in one fixed order on every run.
"""
import pytest

NB = 64            # panel width
BATCH = 8          # panels per batch
BW = BATCH * NB    # batch width in columns
MIN_DIM = 7168     # batched corrections from this size on
RING = 4           # event ring


def plan(d, drop_far_wait=False, short_narrow=False):
    """Ops in enqueue order: (stream, kind, payload); kinds: 'panel' (p),
    'prod' (target 'A' or 'M', first and last block, source panels), 'rec'
    (event name), 'wait' (event name)."""
    ops = []
    n_panels = (d + NB - 1) // NB
    for p in range(n_panels):
        k0 = p * NB
        kb = min(NB, d - k0)
        if p >= 2:
            ops.append(("sp", "wait", ("ev", (p - 2) % RING)))
            ops.append(("sp", "wait", ("ev2", (p - 2) % RING)))
        ops.append(("sp", "panel", p))
        ops.append(("sp", "rec", ("done", 0)))
        ops.append(("s", "wait", ("done", 0)))
        ops.append(("s2", "wait", ("done", 0)))
        b = p // BATCH
        e_b = BATCH * (b + 2) * NB if d >= MIN_DIM else d
        batch_end = p % BATCH == BATCH - 1 and e_b < d
        has_far = batch_end and e_b + BW < d
        r0 = k0 + kb + NB
        c1 = min(e_b, d)
        if short_narrow and c1 < d:
            c1 -= NB
        if r0 < c1:
            ops.append(("s", "prod", ("A", r0, c1, [p])))
            ops.append(("s2", "prod", ("M", r0, c1, [p])))
        if batch_end:
            c0 = (p + 1) * NB - BW
            srcs = list(range(c0 // NB, p + 1))
            e = e_b
            n = min(BW, d - e)
            if b >= 1 and not drop_far_wait:
                ops.append(("s", "wait", ("far", (b - 1) % RING)))
                ops.append(("s2", "wait", ("far2", (b - 1) % RING)))
            ops.append(("s", "prod", ("A", e, e + n, srcs)))
            ops.append(("s2", "prod", ("M", e, e + n, srcs)))
            if has_far:
                f = e + BW
                hb = min(BW, d - f)
                ops.append(("s3", "wait", ("done", 0)))
                ops.append(("s4", "wait", ("done", 0)))
                for part in range(2):
                    g0 = f if part == 0 else f + hb
                    if d - g0 <= 0:
                        break
                    ng = hb if part == 0 else d - g0
                    ops.append(("s3", "prod", ("A", g0, g0 + ng, srcs)))
                    ops.append(("s4", "prod", ("M", g0, g0 + ng, srcs)))
                    if part == 0:
                        ops.append(("s3", "rec", ("far", b % RING)))
                        ops.append(("s4", "rec", ("far2", b % RING)))
        ops.append(("s", "rec", ("ev", p % RING)))
        ops.append(("s2", "rec", ("ev2", p % RING)))
    return ops, n_panels


def graph(ops):
    """Happens-before sets (as bit masks over op indices) of every op."""
    last_on = {}
    last_rec = {}
    before = []
    for i, (st, kind, pay) in enumerate(ops):
        m = 0
        if st in last_on:
            j = last_on[st]
            m |= before[j] | (1 << j)
        if kind == "wait" and pay in last_rec:
            j = last_rec[pay]
            m |= before[j] | (1 << j)
        before.append(m)
        last_on[st] = i
        if kind == "rec":
            last_rec[pay] = i
    return before


def check(d, **mistake):
    ops, n_panels = plan(d, **mistake)
    before = graph(ops)
    panel_at = {pay: i for i, (st, kind, pay) in enumerate(ops) if kind == "panel"}
    for target in ("A", "M"):
        applied = {}
        writers = {}   # block -> op indices of the products writing it
        for i, (st, kind, pay) in enumerate(ops):
            if kind != "prod" or pay[0] != target:
                continue
            _, lo, hi, srcs = pay
            assert lo % NB == 0 and lo < hi <= d
            for cb in range(lo // NB, (hi + NB - 1) // NB):
                writers.setdefault(cb, []).append(i)
                for q in srcs:
                    key = (q, cb)
                    assert key not in applied, f"{target} {key} applied twice (d={d})"
                    applied[key] = i
        for q in range(n_panels):
            for cb in range(q + 2, n_panels):
                assert (q, cb) in applied, f"{target}: panel {q} never reaches block {cb} (d={d})"
        for cb, idx in writers.items():
            for i in idx:
                assert before[panel_at[cb]] >> i & 1, f"{target}: block {cb} written after its panel (d={d})"
            for a in range(len(idx)):
                for c in range(a + 1, len(idx)):
                    i, j = idx[a], idx[c]
                    assert (before[j] >> i & 1) or (before[i] >> j & 1), \
                        f"{target}: unordered writes to block {cb} (d={d})"


@pytest.mark.parametrize("d", [64, 200, 1000, 4096, 7104, 7168, 7232, 7680, 8192, 8256, 11008,
                               12288, 16384, 16448, 20480])
def test_factorisation_plan(d):
    check(d)


def test_factorisation_plan_sweep():
    for d in range(7168 - 512, 14336 + 1, 64 * 7):
        check(d)


def test_the_checks_see_planted_mistakes():
    """A band product that does not wait for the previous far product leaves
    that far product unordered against later panels and products; a narrow
    region one block short leaves a contribution unapplied."""
    with pytest.raises(AssertionError, match="unordered writes|written after its panel"):
        check(11008, drop_far_wait=True)
    with pytest.raises(AssertionError, match="never reaches"):
        check(11008, short_narrow=True)
