"""Host-side check of the specialised kernel's pipeline protocol.

The sm_100a kernel synchronises its roles (halo producer, weight producer,
MMA issuer, epilogue, transform groups) with mbarriers whose waits test a
phase parity.  This test replays that protocol on the CPU for the plans the
library's own planner (q3d_plan_conv, host code) chooses, and checks that
  - no interleaving explored here deadlocks (every role finishes), and
  - every parity wait that succeeds does so for the phase it means, i.e. the
    barrier has completed exactly that phase and not one two phases earlier
    (parity aliasing),
together with the plan invariants the kernel relies on.  Roles are modelled
as generators yielding ("wait", barrier, phase) or ("arrive", barrier);
TMA and tcgen05.commit completions are arrivals issued where the kernel
issues them.  Several schedules (round-robin, reversed, seeded random) are
explored.
"""
import random

import pytest
import torch

from quantized_conv3d_implicit_b200 import api, workloads


class Bar:
    def __init__(self, count):
        self.count, self.pending, self.phase = count, count, 0

    def arrive(self, phase=None):
        # an arrival meant for a given phase must not land in an earlier one
        assert phase is None or phase == self.phase, f"arrival for phase {phase} while at {self.phase}"
        self.pending -= 1
        if self.pending == 0:
            self.phase += 1
            self.pending = self.count

    def parity_done(self, phase):
        return (self.phase & 1) != (phase & 1)


def roles(plan, K, taps, ntiles, kernel="fast", units=None, blk64=False):
    """units (tensor-memory kernel): the CTA's work as (k0, k1) K-slice
    ranges of successive tiles; default ntiles whole tiles.  blk64
    (tensor-memory kernel, NVFP4 blocks of 64): every warp holds all four
    blocks of its rows (lanes l and l + 16 two each), waits for all their
    slots and hands back slots by block 0's position."""
    bars = {}

    def bar(name, i, count):
        key = (name, i)
        if key not in bars:
            bars[key] = Bar(count)
        return bars[key]

    ks, q_slots, ring, sa, sb, G = (plan[k] for k in ("ks", "q_slots", "ring", "sa", "sb", "groups"))
    n_mt, n_sub, c_slot = plan["n_mt"], plan["n_sub"], plan["c_slot"]
    nbuf = plan.get("acc_bufs", 1) or 1   # accumulator buffers (the tensor-memory kernel may have two)
    # tensor-memory kernel: hand-backs wait for each slot's fill first
    hb_wait = bool(plan.get("hb_wait", 0)) or plan["ks"] < plan["sa"]
    n_xf = 16 if kernel == "tmem" else 8   # transform warps; the tensor-memory kernel has one group
    wpg = n_xf // G
    # who hands halo slots back: the MMA thread (shared-memory kernel) or
    # every transform warp once it is past the slot (tensor-memory kernel)
    xf_release = kernel == "tmem"
    halo_empty_count = n_xf if xf_release else 1

    def slot_lo(s):
        return ((64 * s) // taps) // c_slot

    def slot_hi(s):
        return (min(64 * s + 63, K - 1) // taps) // c_slot

    us = units if units is not None else [(0, ks)] * ntiles

    def unit_slots(k0, k1):   # first halo slot of a unit and its slot count
        lo = ((64 * k0) // taps) // c_slot
        return lo, (min(64 * k1, K) - 1) // taps // c_slot - lo + 1

    def halo_producer():
        gs = 0
        for k0, k1 in us:
            for _q in range(unit_slots(k0, k1)[1]):
                e, u = gs % ring, gs // ring
                if u > 0:
                    yield ("wait", bar("halo_empty", e, halo_empty_count), u - 1)
                yield ("arrive", bar("halo_full", e, 1))
                gs += 1

    def weight_producer():
        gb = 0
        for k0, k1 in us:
            for _s in range(k0, k1):
                e, u = gb % sb, gb // sb
                if u > 0:
                    yield ("wait", bar("b_empty", e, 1), u - 1)
                yield ("arrive", bar("b_full", e, 1))
                gb += 1

    def mma():
        ga = gb = gs_base = 0
        for it, (k0, k1) in enumerate(us):
            released = 0
            for s in range(k0, k1):
                ea, eb = ga % sa, gb % sb
                yield ("wait", bar("a_full", ea, 8 if kernel == "tmem" else wpg), ga // sa)
                keep = slot_lo(s + 1) if s + 1 < ks else q_slots
                while not xf_release and released < keep:
                    yield ("arrive", bar("halo_empty", (gs_base + released) % ring, 1))
                    released += 1
                yield ("wait", bar("b_full", eb, 1), gb // sb)
                buf, use = it % nbuf, it // nbuf   # accumulator buffer of this unit, and its earlier uses
                for i in range(n_mt):
                    for ns in range(n_sub):
                        acc = (buf * n_mt + i) * n_sub + ns
                        if s == k0 and use > 0:
                            yield ("wait", bar("acc_empty", acc, 4), use - 1)
                        if s == k1 - 1:
                            yield ("arrive", bar("acc_full", acc, 1))
                yield ("arrive", bar("a_empty", ea, 1))
                yield ("arrive", bar("b_empty", eb, 1))
                ga += 1
                gb += 1
            gs_base += q_slots

    def epilogue():
        for it in range(len(us)):
            buf, use = it % nbuf, it // nbuf
            for i in range(n_mt):
                for ns in range(n_sub):
                    acc = (buf * n_mt + i) * n_sub + ns
                    yield ("wait", bar("acc_full", acc, 1), use)
                    yield ("arrive", bar("acc_empty", acc, 4))

    def transform(w):
        grp = w // wpg
        blk = w >> 2   # tensor-memory kernel: 16-column block of every slice
        ga = gs_base = 0
        for _ in range(ntiles):
            s = (grp + G - ga % G) % G
            released = 0
            while s < ks:
                gsl = ga + s
                ea, ua = gsl % sa, gsl // sa
                if ua > 0:
                    yield ("wait", bar("a_empty", ea, 1), ua - 1)
                if xf_release:
                    # only the slots this warp's block reads
                    k0 = 64 * s + 16 * blk
                    qs = []
                    if k0 < K:
                        c0, phi = divmod(k0, taps)
                        q0, cs0 = divmod(c0, c_slot)
                        split, nvalid = taps - phi, K - k0
                        qs = [q0, q0 + 1] if (split < min(16, nvalid) and cs0 + 1 == c_slot) else [q0]
                else:
                    qs = range(slot_lo(s), slot_hi(s) + 1)
                for q in qs:
                    g = gs_base + q
                    yield ("wait", bar("halo_full", g % ring, 1), g // ring)
                yield ("arrive", bar("a_full", ea, wpg))
                if xf_release:
                    # the tensor-memory kernel's warps hand back the slots below
                    # their next block's slot (phase = use of the ring entry)
                    if s + 1 < ks:
                        k0n = 64 * (s + 1) + 16 * blk
                        keep = min((k0n // taps) // c_slot, q_slots)
                    else:
                        keep = q_slots
                    while released < keep:
                        g = gs_base + released
                        yield ("arrive", bar("halo_empty", g % ring, halo_empty_count), g // ring)
                        released += 1
                s += G
            ga += ks
            gs_base += q_slots

    def transform_tmem(w):
        # tensor-memory kernel: group w >> 3 takes the global slices of its
        # parity; warp w handles blocks b0, b0 + 1 of each, waits for the halo
        # slots those read and hands back the slots below its next pair
        grp, b0 = w >> 3, ((w >> 2) & 1) * 2
        b0s = (0, 2) if blk64 else (b0,)   # the blocks the warp's lanes start at
        b_rel = 0 if blk64 else b0         # lane 0's block: the hand-back position
        gs_base = ga = 0
        gslice = grp
        hr = 0  # next global slot to hand back
        for k0u, k1u in us:
            q_lo, n_q = unit_slots(k0u, k1u)
            s = k0u + gslice - ga
            released = 0
            while s < k1u:
                ea, ua = gslice % sa, gslice // sa
                if gslice >= sa:
                    yield ("wait", bar("a_empty", ea, 1), ua - 1)
                for bw in b0s:
                    k0 = 64 * s + 16 * bw
                    if k0 >= K:
                        continue
                    c0, phi = divmod(k0, taps)
                    q0, cs0 = divmod(c0, c_slot)
                    c1, phi1 = divmod(k0 + 16, taps)
                    q1, cs1 = divmod(c1, c_slot)
                    nv0, nv1 = K - k0, K - k0 - 16
                    aligned = (c_slot * taps) % 16 == 0   # no block straddles two slots
                    cross0 = not aligned and (taps - phi) < min(16, nv0) and cs0 + 1 == c_slot
                    cross1 = not aligned and (taps - phi1) < min(16, nv1) and cs1 + 1 == c_slot
                    q_last = q1 + int(cross1) if nv1 > 0 else q0 + int(cross0)
                    for q in range(q0, q_last + 1):
                        assert q_lo <= q < q_lo + n_q, "a block reads a slot outside its unit"
                        g = gs_base + q - q_lo
                        yield ("wait", bar("halo_full", g % ring, 1), g // ring)
                yield ("arrive", bar("a_full", ea, 8))
                if s + 2 < k1u:
                    keep = min(((64 * (s + 2) + 16 * b_rel) // taps) // c_slot - q_lo, n_q)
                else:
                    keep = n_q
                while released < keep:
                    # with ks < sa, sa slices span several tiles' slots and a
                    # warp hands back slots it never read: it waits for each
                    # slot's fill first so it cannot do so a ring lap early
                    if hb_wait:
                        yield ("wait", bar("halo_full", hr % ring, 1), hr // ring)
                    yield ("arrive", bar("halo_empty", hr % ring, 16), hr // ring)
                    released += 1
                    hr += 1
                s += 2
                gslice += 2
            while released < n_q:
                # with ks < sa a slot handed back at the end of a tile waits
                # for its fill first: a warp with no slice in the tile would
                # otherwise run a ring lap ahead and arrive in an earlier phase
                if hb_wait:
                    yield ("wait", bar("halo_full", hr % ring, 1), hr // ring)
                yield ("arrive", bar("halo_empty", hr % ring, 16), hr // ring)
                released += 1
                hr += 1
            gs_base += n_q
            ga += k1u - k0u

    r = {"halo": halo_producer(), "weights": weight_producer(), "mma": mma()}
    for w in range(4):
        r[f"epilogue{w}"] = epilogue()
    for w in range(n_xf):
        r[f"transform{w}"] = transform_tmem(w) if kernel == "tmem" else transform(w)
    return r


def run(plan, K, taps, ntiles, order="rr", seed=0, kernel="fast", units=None, blk64=False):
    rs = roles(plan, K, taps, ntiles, kernel, units, blk64)
    names = list(rs)
    cur = {k: None for k in names}
    done = set()
    rng = random.Random(seed)
    while len(done) < len(names):
        progress = False
        seq = names if order == "rr" else names[::-1] if order == "rev" else rng.sample(names, len(names))
        for k in seq:
            if k in done:
                continue
            steps = 0
            while order != "random" or steps < rng.randint(1, 4):
                steps += 1
                if cur[k] is None:
                    try:
                        cur[k] = next(rs[k])
                    except StopIteration:
                        done.add(k)
                        progress = True
                        break
                op = cur[k]
                if op[0] == "arrive":
                    op[1].arrive(op[2] if len(op) > 2 else None)
                    cur[k] = None
                    progress = True
                    continue
                b, phase = op[1], op[2]
                if b.parity_done(phase):
                    assert b.phase == phase + 1, f"parity aliasing in {k}: waits phase {phase}, barrier at {b.phase}"
                    cur[k] = None
                    progress = True
                    continue
                break
        assert progress, "deadlock: " + ", ".join(k for k in names if k not in done)


def _plan(wl_or_args, kernel="fast"):
    if isinstance(wl_or_args, workloads.Workload):
        wl = wl_or_args
        pad6 = (wl.pad_lo[0], wl.pad_hi[0], wl.pad_lo[1], wl.pad_hi[1], wl.pad_lo[2], wl.pad_hi[2])
        w_shape = (wl.cout, wl.x_shape[1]) + tuple(wl.kernel)
        return api.plan_conv(wl.x_shape, w_shape, wl.stride, pad6, wl.dil, wl.dtype, kernel=kernel), wl.k_gemm, \
            wl.kernel[0] * wl.kernel[1] * wl.kernel[2]
    xs, ws, s, pad6, d, dt = wl_or_args
    return api.plan_conv(xs, ws, s, pad6, d, dt, kernel=kernel), ws[1] * ws[2] * ws[3] * ws[4], \
        ws[2] * ws[3] * ws[4]


def _check_invariants(p):
    assert p["sa"] >= p["groups"]
    assert p["groups"] == (1 if p["n_mt"] >= 4 else 2)
    assert p["n_mt"] * p["n_tile"] <= p["tmem_cols"] <= 512
    assert p["n_sub"] * p["sub_n"] == p["n_tile"] and p["sub_n"] % 16 == 0 and 16 <= p["sub_n"] <= 256
    assert p["smem"] <= 232448
    assert p["TH"] * p["TW"] == 128
    assert p["w_box"] <= 256 and p["h_ext"] <= 256 and p["kd_ext"] <= 256


@pytest.mark.parametrize("name", sorted(workloads.WORKLOADS))
@pytest.mark.parametrize("order", ["rr", "rev", "random"])
def test_workload_plans_are_deadlock_and_alias_free(name, order):
    plan, K, taps = _plan(workloads.WORKLOADS[name])
    assert plan["applicable"] == 1
    _check_invariants(plan)
    run(plan, K, taps, ntiles=3, order=order, seed=sum(map(ord, name)))


def test_random_shapes():
    rng = random.Random(7)
    checked = 0
    for _ in range(60):
        k = rng.choice([(1, 1, 1), (3, 3, 3), (1, 3, 3), (5, 5, 5), (3, 1, 1)])
        cin = rng.choice([1, 3, 8, 16, 37, 64, 96, 192, 256])
        cout = rng.choice([1, 8, 16, 40, 96, 100, 192, 256, 300, 384, 512, 640, 1024])
        xs = (rng.choice([1, 2]), cin, rng.randint(k[0], 9), rng.randint(k[1], 40), 8 * rng.randint(1, 30))
        s = (1, rng.choice([1, 1, 2]), rng.choice([1, 1, 2]))
        d = (1, rng.choice([1, 2]), rng.choice([1, 2]))
        pad6 = tuple(rng.randint(0, 2) for _ in range(6))
        ws = (cout, cin) + k
        dt = rng.choice([torch.bfloat16, torch.float16, torch.float32])
        try:
            plan, K, taps = _plan((xs, ws, s, pad6, d, dt))
        except api.Q3DError:
            continue  # empty output: not a valid convolution
        if not plan["applicable"]:
            continue
        _check_invariants(plan)
        run(plan, K, taps, ntiles=2, order="random", seed=checked)
        checked += 1
    assert checked >= 30


def test_sim_detects_aliasing_when_stages_fewer_than_groups():
    # the checker itself: with fewer A stages than transform groups a group can
    # pass a wait two phases early, which the model must flag
    plan, K, taps = _plan(workloads.WORKLOADS["wan_mid_384_bf16"])
    assert plan["groups"] >= 2
    bad = dict(plan, sa=plan["groups"] - 1)
    with pytest.raises(AssertionError):
        run(bad, K, taps, ntiles=3)


def _check_tmem_invariants(p, taps):
    assert p["groups"] == 2 and p["tmem_cols"] == 512
    if taps < 16:
        # a block spans several channels: slots must hold whole blocks
        assert (p["c_slot"] * taps) % 16 == 0
    nb = p["acc_bufs"]
    assert nb in (1, 2) and p["aop"] in (0, 1) and p["sa"] >= 2
    if p["aop"] == 0:
        # acc_bufs accumulators [0, nb*n_mt*n_tile), then sa A stages of n_mt * 32 columns
        assert nb * p["n_mt"] * p["n_tile"] <= p["a_col0"] and p["a_col0"] % 32 == 0
        assert p["a_col0"] + p["sa"] * p["n_mt"] * 32 <= 512
    else:
        # A in shared memory: tensor memory holds only the accumulators
        assert nb * p["n_mt"] * p["n_tile"] <= 512
    assert nb * p["n_mt"] * p["n_sub"] <= 16
    assert p["n_sub"] * p["sub_n"] == p["n_tile"] and p["sub_n"] % 16 == 0 and 16 <= p["sub_n"] <= 256
    assert p["smem"] <= 232448 and p["TH"] * p["TW"] == 128
    assert p["w_box"] <= 256 and p["h_ext"] <= 256 and p["kd_ext"] <= 256


@pytest.mark.parametrize("name", sorted(workloads.WORKLOADS))
@pytest.mark.parametrize("order", ["rr", "rev", "random"])
def test_tmem_kernel_plans_are_deadlock_and_alias_free(name, order):
    plan, K, taps = _plan(workloads.WORKLOADS[name], kernel="tmem")
    assert plan["applicable"] == 1
    _check_tmem_invariants(plan, taps)
    run(plan, K, taps, ntiles=3, order=order, seed=sum(map(ord, name)), kernel="tmem")


def test_tmem_kernel_random_shapes():
    rng = random.Random(11)
    checked = 0
    for _ in range(80):
        k = rng.choice([(3, 3, 3), (5, 5, 5), (3, 3, 2), (1, 5, 5), (2, 3, 3), (1, 1, 1), (1, 3, 3), (3, 1, 1),
                        (2, 2, 2), (1, 2, 2)])
        cin = rng.choice([1, 3, 8, 16, 37, 64, 96, 192, 256])
        cout = rng.choice([1, 8, 16, 40, 96, 100, 192, 256, 300, 384, 448, 512, 640, 1024])
        xs = (rng.choice([1, 2]), cin, rng.randint(k[0], 9), rng.randint(k[1], 40), 8 * rng.randint(1, 30))
        s = (1, rng.choice([1, 1, 2]), rng.choice([1, 1, 2]))
        d = (1, rng.choice([1, 2]), rng.choice([1, 2]))
        pad6 = tuple(rng.randint(0, 2) for _ in range(6))
        ws = (cout, cin) + k
        dt = rng.choice([torch.bfloat16, torch.float16, torch.float32])
        try:
            plan, K, taps = _plan((xs, ws, s, pad6, d, dt), kernel="tmem")
        except api.Q3DError:
            continue  # empty output: not a valid convolution
        if not plan["applicable"]:
            continue
        _check_tmem_invariants(plan, taps)
        run(plan, K, taps, ntiles=2, order="random", seed=checked, kernel="tmem")
        checked += 1
    assert checked >= 40


@pytest.mark.parametrize("kshape", [(1, 1, 1), (1, 3, 3), (3, 1, 1), (2, 2, 2)])
def test_tmem_kernel_plans_blocks_within_one_slot_below_16_taps(kshape):
    taps = kshape[0] * kshape[1] * kshape[2]
    plan, K, _ = _plan(((1, 64, 4, 16, 16), (64, 64) + kshape, 1, 0, 1, torch.bfloat16), kernel="tmem")
    assert plan["applicable"] == 1
    assert (plan["c_slot"] * taps) % 16 == 0
    run(plan, K, taps, ntiles=2, order="rr", kernel="tmem")


def test_tmem_kernel_declines_unaligned_rows():
    plan, _, _ = _plan(((1, 8, 4, 16, 12), (8, 8, 3, 3, 3), 1, 1, 1, torch.bfloat16), kernel="tmem")
    assert plan["applicable"] == 0 and plan["TW"] == 0


@pytest.mark.parametrize("order", ["rr", "rev", "random"])
def test_tmem_kernel_single_slice_tiles_do_not_lap_the_ring(order):
    """One K slice per tile: the second transform group never builds, yet
    hands every slot back; seven tiles of four slots on an 11-slot ring."""
    plan, K, taps = _plan(((1, 64, 32, 64, 256), (32, 64, 1, 1, 1), 1, 0, 1, torch.bfloat16), kernel="tmem")
    assert plan["ks"] == 1 and 7 * plan["q_slots"] > 2 * plan["ring"]
    run(plan, K, taps, 7, order=order, seed=5, kernel="tmem")


@pytest.mark.parametrize("shape", [((1, 96, 3, 16, 64), 96), ((1, 384, 5, 60, 104), 384), ((1, 11, 4, 7, 16), 41),
                                   ((1, 3, 7, 9, 16), 8), ((1, 96, 17, 480, 832), 96)])
@pytest.mark.parametrize("order", ["rr", "rev", "random"])
def test_tmem_kernel_blocks_of_64_lane_pairs(shape, order, monkeypatch):
    """NVFP4 blocks of 64 (A in shared memory, the plan the launcher forces):
    each warp waits for the slots of all four blocks of its rows and hands
    back by block 0's position; no interleaving deadlocks or aliases."""
    monkeypatch.setenv("Q3D_KERNEL", "smem_a")
    xs, cout = shape
    k = (5, 5, 5) if xs[1] == 3 else (3, 3, 3)
    plan, K, taps = _plan((xs, (cout, xs[1]) + k, 1, (2, 0, 1, 1, 1, 1), 1, torch.bfloat16), kernel="tmem")
    assert plan["applicable"] == 1 and plan["aop"] == 1
    run(plan, K, taps, ntiles=3, order=order, seed=len(xs) + cout, kernel="tmem", blk64=True)


@pytest.mark.parametrize("name", sorted(workloads.WORKLOADS))
@pytest.mark.parametrize("order", ["rr", "rev", "random"])
def test_tmem_kernel_forced_shared_memory_plans(name, order, monkeypatch):
    """A in shared memory where the launcher would not choose it (forced, as
    the GPU tests and blocks of 64 do): the plan's hand-backs wait for the
    fills, and no interleaving deadlocks or aliases, for the default mapping
    and for the blocks-of-64 lane pairs."""
    monkeypatch.setenv("Q3D_KERNEL", "smem_a")
    plan, K, taps = _plan(workloads.WORKLOADS[name], kernel="tmem")
    assert plan["applicable"] == 1 and plan["aop"] == 1
    for blk64 in (False, True):
        run(plan, K, taps, ntiles=3, order=order, seed=sum(map(ord, name)), kernel="tmem", blk64=blk64)


def _plan_fp4(xs, ws, s, pad6, d, dt):
    p = api.plan_conv(xs, ws, s, pad6, d, dt, kernel="fp4")
    return p, ws[1] * ws[2] * ws[3] * ws[4], ws[2] * ws[3] * ws[4]


@pytest.mark.parametrize("name", sorted(workloads.WORKLOADS))
@pytest.mark.parametrize("order", ["rr", "rev", "random"])
def test_fp4_variant_plans_are_deadlock_and_alias_free(name, order):
    """The NVFP4-operand form keeps the roles and barriers (its MMA warp
    also copies scale factors, which the commits already order): its plans
    replayed like the BF16 ones."""
    wl = workloads.WORKLOADS[name]
    ws = (wl.cout, wl.x_shape[1]) + tuple(wl.kernel)
    pad6 = (wl.pad_lo[0], wl.pad_hi[0], wl.pad_lo[1], wl.pad_hi[1], wl.pad_lo[2], wl.pad_hi[2])
    plan, K, taps = _plan_fp4(wl.x_shape, ws, wl.stride, pad6, wl.dil, wl.dtype)
    assert plan["applicable"] == 1
    run(plan, K, taps, ntiles=3, order=order, seed=sum(map(ord, name)), kernel="tmem")


def test_fp4_variant_random_shapes():
    rng = random.Random(3)
    checked = 0
    for _ in range(80):
        k = rng.choice([(3, 3, 3), (5, 5, 5), (1, 1, 1), (1, 3, 3), (3, 1, 1), (2, 2, 2)])
        cin = rng.choice([1, 3, 8, 16, 37, 64, 96, 192])
        cout = rng.choice([8, 16, 40, 96, 192, 256, 384, 512, 1024])
        xs = (rng.choice([1, 2]), cin, rng.randint(k[0], 9), rng.randint(k[1], 40), 8 * rng.randint(1, 30))
        dt = rng.choice([torch.bfloat16, torch.float16, torch.float32])
        try:
            plan, K, taps = _plan_fp4(xs, (cout, cin) + k, 1, (1, 1, 1, 1, 1, 1), 1, dt)
        except api.Q3DError:
            continue
        if not plan["applicable"]:
            continue
        run(plan, K, taps, ntiles=2, order="random", seed=checked, kernel="tmem")
        checked += 1
    assert checked >= 40


def test_tmem_kernel_forced_shared_memory_random_shapes(monkeypatch):
    """Random shapes with A in shared memory forced (the GPU tests' smem_a
    switch, blocks of 64): deadlock- and alias-free for both lane mappings."""
    monkeypatch.setenv("Q3D_KERNEL", "smem_a")
    rng = random.Random(19)
    checked = 0
    for _ in range(80):
        k = rng.choice([(3, 3, 3), (5, 5, 5), (1, 1, 1), (1, 3, 3), (3, 1, 1), (2, 2, 2)])
        cin = rng.choice([1, 3, 8, 16, 37, 64, 96, 192, 256])
        cout = rng.choice([1, 8, 16, 40, 96, 100, 192, 256, 300, 384, 448, 512, 1024])
        xs = (rng.choice([1, 2]), cin, rng.randint(k[0], 9), rng.randint(k[1], 40), 8 * rng.randint(1, 30))
        s = (1, rng.choice([1, 1, 2]), rng.choice([1, 1, 2]))
        d = (1, rng.choice([1, 2]), rng.choice([1, 2]))
        pad6 = tuple(rng.randint(0, 2) for _ in range(6))
        dt = rng.choice([torch.bfloat16, torch.float16, torch.float32])
        try:
            plan, K, taps = _plan((xs, (cout, cin) + k, s, pad6, d, dt), kernel="tmem")
        except api.Q3DError:
            continue
        if not plan["applicable"] or plan["aop"] != 1:
            continue
        for blk64 in (False, True):
            run(plan, K, taps, ntiles=2, order="random", seed=checked, kernel="tmem", blk64=blk64)
        checked += 1
    assert checked >= 30
