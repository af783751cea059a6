"""The host-side execution plan of a decoder stack (CPU only, no CUDA call).

lb_stack_plan_host writes the plan lb_stack_prepare would put in a workspace
into a host image.  These tests check what the decode kernel relies on:
- every phase's split table covers its units once, in order;
- the units of a phase map one-to-one onto (job, slice, rowblock), and each
  CTA's start record is the first batch of its range under that mapping;
- each phase zeroes exactly the accumulators the next phase adds into.
"""
import ctypes

import numpy as np
import pytest

from binary_rank_linear_lb_b200.configs import LLAMA2_13B, LLAMA2_70B, Model

TAG_X, TAG_Y = 1, 2            # the call's x and y, stored as tags in the plan
K_TABLES = 2                   # tiles of one batch (tables resident at once)

PHASE = np.dtype([("job_begin", "<i4"), ("n_jobs", "<i4"), ("n_units", "<i4"), ("zero_n", "<i4"),
                  ("zero_ptr", "<u8"), ("split_off", "<i4"), ("split_g", "<i4"),
                  ("next_job_begin", "<i4"), ("next_n_jobs", "<i4"), ("starts_g", "<i4"),
                  ("pad", "<i4")])
JOB = np.dtype([("P", "<u8"), ("src", "<u8"), ("src2", "<u8"), ("vscale", "<u8"),
                ("oscale", "<u8"), ("out", "<u8"), ("norm_sumsq", "<u8"), ("acc_sumsq", "<u8"),
                ("resid_init", "<u8"), ("rows", "<i4"), ("cols", "<i4"), ("ldw", "<i4"),
                ("kind", "<i4"), ("n_slices", "<i4"), ("n_rowblocks", "<i4"),
                ("unit_begin", "<i4"), ("norm_n", "<i4"), ("gqa_ghd", "<i4"), ("gqa_hd", "<i4"),
                ("rg", "<i4"), ("sliced", "<i4"), ("pad", "<i4", (2,))])
START = np.dtype([("u", "<i4"), ("u_end", "<i4"), ("j", "<i4"), ("nt", "<i4"), ("n_rb", "<i4"),
                  ("pad", "<i4", (3,)), ("t", "<i4", (2, 4))])

SMALL = Model("small", hidden=256, inter=512, n_heads=4, n_kv_heads=2, head_dim=64, n_layers=3)
SMALL_RANKS = [64, 32, 32, 64, 96, 96, 96]


@pytest.fixture(scope="module")
def lb():
    from binary_rank_linear_lb_b200 import build
    build.build()
    import binary_rank_linear_lb_b200 as m
    return m


def plan(lb, model, bpw, n_layers, grid, mlp_only=False):
    ranks = SMALL_RANKS if model is SMALL else model.ranks(bpw)
    return plan_ranks(lb, model, ranks, n_layers, grid, mlp_only)


def plan_ranks(lb, model, ranks, n_layers, grid, mlp_only=False):
    """(phases, jobs, split rows, start rows, image base, accumulator end) of a stack
    whose packed factors sit at made-up aligned addresses (the planner never reads them)."""
    nb = 2
    n = n_layers * 7 * nb
    fake = lambda i: 1 << 40 | i << 12
    brs = (lb.lb_branch * n)(*[lb.lb_branch(fake(5 * i), fake(5 * i + 1), fake(5 * i + 2),
                                            fake(5 * i + 3), fake(5 * i + 4))
                               for i in range(n)])
    for b in brs:
        b.layout = lb.LB_LAYOUT_SLICES
    rk = (ctypes.c_int64 * (n_layers * 7))(*(ranks * n_layers))
    d = lb.lb_stack_desc(n_layers, model.hidden, model.inter, model.n_heads, model.n_kv_heads,
                         model.head_dim, nb, lb.LB_STACK_MLP_ONLY if mlp_only else 0,
                         ctypes.addressof(brs), ctypes.addressof(rk))
    L = lb.lib()
    size = L.lb_stack_workspace_size(ctypes.byref(d))
    assert size > 0
    raw = np.zeros(size + 256, dtype=np.uint8)
    base = (raw.ctypes.data + 255) // 256 * 256
    img = raw[base - raw.ctypes.data:][:size]
    offs = (ctypes.c_size_t * 5)()
    cnt = (ctypes.c_int * 6)()
    st = L.lb_stack_plan_host(ctypes.byref(d), grid, ctypes.c_void_p(base), size, offs, cnt)
    assert st == lb.LB_OK, lb.status_string(st)
    n_ph, n_jobs, stride = cnt[0], cnt[1], cnt[2]
    assert (cnt[3], cnt[4], cnt[5]) == (PHASE.itemsize, JOB.itemsize, START.itemsize)
    phases = np.frombuffer(img[offs[0]:], dtype=PHASE, count=n_ph)
    jobs = np.frombuffer(img[offs[1]:], dtype=JOB, count=n_jobs)
    split = np.frombuffer(img[offs[2]:], dtype="<i4", count=n_ph * (stride + 1)).reshape(n_ph, -1)
    starts = np.frombuffer(img[offs[3]:], dtype=START, count=n_ph * stride).reshape(n_ph, -1)
    return phases, jobs, split, starts, base, offs[4]


def next_tile(J, j, u, u_end):
    """The tile of a range starting at unit u: a job's units run row group by row group,
    slice by slice inside a group, rowblock by rowblock inside a slice."""
    while j + 1 < len(J) and J[j + 1]["unit_begin"] <= u:
        j += 1
    job = J[j]
    local = u - job["unit_begin"]
    rg, ns, nrb = int(job["rg"]), int(job["n_slices"]), int(job["n_rowblocks"])
    g, off = divmod(local, rg * ns)
    rows_g = min(rg, nrb - g * rg)
    s, rbi = divmod(off, rows_g)
    return j, (j, s, g * rg + rbi, min(rows_g - rbi, u_end - u))


CASES = [(SMALL, 1.0, 3, 148), (SMALL, 1.0, 3, 7), (LLAMA2_13B, 0.55, 2, 148),
         (LLAMA2_70B, 1.0, 2, 148), (LLAMA2_70B, 0.55, 1, 132)]


@pytest.mark.parametrize("model,bpw,n_layers,grid", CASES)
def test_splits_cover_each_phase_once(lb, model, bpw, n_layers, grid):
    phases, jobs, split, starts, base, acc_end = plan(lb, model, bpw, n_layers, grid)
    assert len(phases) == 8 * n_layers
    for q, ph in enumerate(phases):
        J = jobs[ph["job_begin"]:ph["job_begin"] + ph["n_jobs"]]
        assert 1 <= ph["n_jobs"] <= 16
        # the jobs' units are consecutive and add up to the phase's
        assert J[0]["unit_begin"] == 0
        sizes = J["n_slices"].astype(np.int64) * J["n_rowblocks"]
        assert (np.diff(J["unit_begin"]) == sizes[:-1]).all()
        assert sizes.sum() == ph["n_units"]
        assert ((J["rg"] >= 1) & (J["rg"] <= J["n_rowblocks"])).all()
        # the split: G+1 non-decreasing boundaries from 0 to n_units
        assert ph["split_g"] == grid
        sp = split[q][:grid + 1]
        assert sp[0] == 0 and sp[-1] == ph["n_units"]
        assert (np.diff(sp) >= 0).all()
        assert ph["next_n_jobs"] == (phases[q + 1]["n_jobs"] if q + 1 < len(phases) else 0)


@pytest.mark.parametrize("model,bpw,n_layers,grid", CASES)
def test_units_map_one_to_one_and_start_records_match(lb, model, bpw, n_layers, grid):
    phases, jobs, split, starts, base, acc_end = plan(lb, model, bpw, n_layers, grid)
    for q, ph in enumerate(phases):
        J = jobs[ph["job_begin"]:ph["job_begin"] + ph["n_jobs"]]
        seen = set()
        for c in range(grid):
            u, u_end = int(split[q][c]), int(split[q][c + 1])
            S = starts[q][c]
            assert ph["starts_g"] == grid
            assert (S["u"], S["u_end"]) == (u, u_end)
            j, first, k = 0, [], 0
            while u < u_end:
                j, t = next_tile(J, j, u, u_end)
                assert t[3] >= 1
                if len(first) < K_TABLES and u - S["u"] == sum(x[3] for x in first):
                    first.append(t)
                for rb in range(t[2], t[2] + t[3]):
                    key = (t[0], t[1], rb)
                    assert key not in seen
                    seen.add(key)
                u += t[3]
            assert S["nt"] == len(first)
            assert S["n_rb"] == sum(t[3] for t in first)
            for k, t in enumerate(first):
                assert tuple(S["t"][k]) == t
        want = {(j, s, rb) for j in range(len(J)) for s in range(J[j]["n_slices"])
                for rb in range(J[j]["n_rowblocks"])}
        assert seen == want


@pytest.mark.parametrize("model,bpw,n_layers,grid", CASES[:4])
def test_each_phase_zeroes_what_the_next_one_adds_into(lb, model, bpw, n_layers, grid):
    phases, jobs, split, starts, base, acc_end = plan(lb, model, bpw, n_layers, grid)
    n = len(phases)
    for q in range(n):
        nxt = phases[(q + 1) % n]
        zp, zn = int(phases[q]["zero_ptr"]), int(phases[q]["zero_n"])
        lo, hi = (zp - base, zp - base + 4 * zn) if zp else (0, 0)
        if zp:
            assert 256 <= lo <= hi <= acc_end
        J = jobs[nxt["job_begin"]:nxt["job_begin"] + nxt["n_jobs"]]
        for job in J:
            for f, n_f in (("out", job["rows"]), ("acc_sumsq", 1)):
                p = int(job[f])
                if p in (0, TAG_X, TAG_Y):
                    continue
                off = p - base
                assert lo <= off and off + 4 * n_f <= hi, (q, f, off, lo, hi)
    # the regions of different phases do not overlap
    ranges = sorted((int(ph["zero_ptr"]) - base, int(ph["zero_ptr"]) - base + 4 * int(ph["zero_n"]))
                    for ph in phases if ph["zero_ptr"])
    for (a0, a1), (b0, b1) in zip(ranges, ranges[1:]):
        assert a1 <= b0


def test_grid_beyond_the_tables_leaves_the_split_to_the_device(lb):
    phases, jobs, split, starts, base, acc_end = plan(lb, SMALL, 1.0, 1, 300)
    assert (phases["starts_g"] == -1).all()
    assert (phases["split_g"] != 300).all()
