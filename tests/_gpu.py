"""Helpers shared by the GPU parity tests: run the CUDA path through the C ABI and compare it
with the CPU oracle on the same seeded inputs."""
import numpy as np
import torch

from oracle import attention as OA
from oracle import schedule as OS
from tests._util import anchors_per_sample, oracle_problem, to_np

# Tolerances. The stated bar is max-abs 2e-2 for bf16 and 1e-4 relative (to max|ref|) for fp32.
# Attention outputs over tens of thousands of keys are small (|O| ~ 1e-2), so an absolute bound
# alone would pass an all-zero result; every float comparison therefore also bounds the error
# relative to the tensor's largest reference value (bf16: P and O are rounded to 8-bit mantissas,
# 2^-9 per rounding; the bound leaves ~10x headroom).
BF16_ABS = 2e-2
BF16_REL = 2e-2
F32_REL = 1e-4


def counts_of(inp):
    off = inp.anchor_off.tolist()
    return [off[i + 1] - off[i] for i in range(len(off) - 1)]


def run_forward(inp, n_workers=None, flags=0, device="cuda"):
    from split_kv_lse_splitkv_b200 import SplitKV
    w = inp.workload
    nw = n_workers if n_workers is not None else w.n_workers
    skv = SplitKV(w.seq_lens, counts_of(inp), w.n_q_heads, w.n_kv_heads, w.head_dim, w.block, w.chunk, w.key_tile,
                  w.scale, w.torch_dtype, n_workers=nw, device=device, blocks_per_item=w.blocks_per_item,
                  chunks_per_item=w.chunks_per_item, item_overhead=w.item_overhead)
    dev = {k: getattr(inp, k).to(device) for k in ("q", "k", "v", "kb", "vb")}
    anchors = inp.anchors.to(device)
    o, lse = skv.forward(dev["q"], dev["k"], dev["v"], dev["kb"], dev["vb"], anchors, flags=flags)
    torch.cuda.synchronize()
    return skv, dev, anchors, o, lse


def assert_close(name, got, ref, dtype, magnitude_scaled=False):
    """Max error within the bound of `dtype`; prints the measured error, the bound and max|ref| so the
    headroom shows in the test log.

    magnitude_scaled (O tensors only): inputs deliberately far from the workloads' N(0,1) scale, e.g.
    rows dominated by one key of 12x the norm, where |O| reaches the size of a single V row. The bf16
    absolute bound is then 2e-2 x max(1, max|ref|): the path rounds to bf16 three times (P before the
    PV product, the stored partial O_c, the output O), each within 2^-9 of the value rounded, so the
    rounding error alone grows with |O| (at most 3 x 2^-9 x max|V|, before any accumulation error).
    LSE is float32 from float32 row sums and is never scaled."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (name, got.shape, ref.shape)
    assert np.isfinite(got).all(), f"{name}: non-finite values"
    err = float(np.max(np.abs(got - ref))) if got.size else 0.0
    scale = float(np.max(np.abs(ref))) if ref.size else 0.0
    if dtype == "f32":
        bound = F32_REL * scale + 1e-30
        print(f"[parity] {name}: max err {err:.3e}, bound {bound:.3e} (f32 rel), max|ref| {scale:.3e}")
        assert err <= bound, f"{name}: max err {err:.3e} > {F32_REL} x {scale:.3e}"
    else:
        if magnitude_scaled:
            assert not name.startswith("LSE"), "LSE keeps the plain absolute bound"
        bound = BF16_ABS * (max(1.0, scale) if magnitude_scaled else 1.0)
        print(f"[parity] {name}: max abs err {err:.3e}, bound {bound:.3e} (bf16 abs), "
              f"rel bound {BF16_REL * scale:.3e}, max|ref| {scale:.3e}")
        assert err <= bound, f"{name}: max abs err {err:.3e} > {bound:.3e}"
        assert err <= BF16_REL * scale + 1e-30, f"{name}: max err {err:.3e} > {BF16_REL} x max|ref| {scale:.3e}"
    return err, scale


def check_cost_and_plan(skv, inp):
    """Costs, compacted item list, chunk costs and the LPT plan must equal the oracle bit for bit."""
    w = inp.workload
    ids, costs, chunk_costs = OS.costs_closed_form(anchors_per_sample(inp), w.seq_lens, w.chunk, w.key_tile,
                                                   w.n_kv_heads, pack=w.blocks_per_item, runs=w.chunks_per_item,
                                                   overhead=w.item_overhead)
    n = int(skv.n_items.item())
    assert n == len(ids)
    assert skv.item_id[:n].cpu().numpy().tolist() == ids.tolist()
    assert skv.item_cost[:n].cpu().numpy().tolist() == costs.tolist()
    assert skv.chunk_cost[:len(chunk_costs)].cpu().numpy().tolist() == chunk_costs.tolist()
    iw, qo, qi, load = OS.lpt(costs.tolist(), skv.n_workers)
    assert skv.item_worker[:n].cpu().numpy().tolist() == iw.tolist()
    assert skv.queue_off.cpu().numpy().tolist() == qo.tolist()
    assert skv.queue_items[:n].cpu().numpy().tolist() == qi.tolist()
    assert skv.load.cpu().numpy().tolist() == load.tolist()
    return ids, costs


def check_partials(skv, inp, ids, magnitude_scaled=False):
    """Every visible item's partial (O_c, LSE_c), and every block's self partial over its own keys,
    against the oracle's chunk-local softmax."""
    w = inp.workload
    p = oracle_problem(inp)
    # One partial per item: over a run of chunks_per_item chunks (the oracle's chunk partials at that size).
    parts = OA.chunk_partials(p, w.chunk * w.chunks_per_item)
    O_part, L_part = skv.o_part_view()
    O_part = O_part.float().cpu().numpy()
    L_part = L_part.cpu().numpy()
    G, R, P = w.group, w.block * w.group, w.blocks_per_item
    RT = int(skv.sizes.rows_per_item)  # rows of a partial tile: P blocks of R rows
    nb = counts_of(inp)
    layout, _ = OS.item_layout(nb, w.seq_lens, w.chunk, w.n_kv_heads, P, w.chunks_per_item)
    bases = [x[0] for x in layout]
    got_O, ref_O, got_L, ref_L = [], [], [], []
    off = inp.anchor_off.tolist()
    anchors = inp.anchors.tolist()
    for item in ids.tolist():
        s = max(i for i in range(len(bases)) if bases[i] <= item)
        nt = layout[s][2]
        local = item - bases[s]
        t = local % nt
        c = (local // nt) // w.n_kv_heads
        g = (local // nt) % w.n_kv_heads
        o_tile = O_part[item].transpose(1, 0, 2).reshape(RT, -1)  # [rows, d]
        for x in range(min(P, nb[s] - t * P)):
            j = off[s] + t * P + x
            if anchors[j] <= c * w.chunk * w.chunks_per_item:
                continue  # this block of the tile sees no key of the chunk (its rows hold O = 0, LSE = -inf)
            for hl in range(G):
                ref_o, ref_l = parts[(s, c, j, g * G + hl)]
                rows = [x * R + i * G + hl for i in range(w.block)]
                got_O.append(o_tile[rows])
                ref_O.append(ref_o)
                got_L.append(L_part[item][rows])
                ref_L.append(ref_l)
    assert bool(got_O) == (len(ids) > 0), "every problem with items has visible chunk partials to compare"
    if got_O:
        assert_close("O_part", np.stack(got_O), np.stack(ref_O), w.dtype, magnitude_scaled)
        assert_close("LSE_part", np.stack(got_L), np.stack(ref_L), w.dtype)
    n_max = int(skv.sizes.n_items_max)
    got_O, ref_O, got_L, ref_L = [], [], [], []
    for s in range(len(w.seq_lens)):
        for j in range(off[s], off[s + 1]):
            for g in range(w.n_kv_heads):
                slot = n_max + j * w.n_kv_heads + g
                o_tile = O_part[slot].transpose(1, 0, 2).reshape(RT, -1)
                for hl in range(G):
                    ref_o, ref_l = parts[(s, -1, j, g * G + hl)]
                    rows = [i * G + hl for i in range(w.block)]
                    got_O.append(o_tile[rows])
                    ref_O.append(ref_o)
                    got_L.append(L_part[slot][rows])
                    ref_L.append(ref_l)
    if got_O:
        assert_close("O_self", np.stack(got_O), np.stack(ref_O), w.dtype, magnitude_scaled)
        assert_close("LSE_self", np.stack(got_L), np.stack(ref_L), w.dtype)
