"""Test helpers: turn seeded workload inputs into oracle problems, and read golden fixtures."""
import os

import numpy as np
import torch

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def to_np(t):
    return None if t is None else t.detach().to("cpu", torch.float64).numpy()


def oracle_problem(inp):
    from oracle.attention import Problem
    w = inp.workload
    return Problem(inp.anchors.numpy(), inp.anchor_off.numpy(), inp.key_off.numpy(),
                   to_np(inp.q), to_np(inp.k), to_np(inp.v), to_np(inp.kb), to_np(inp.vb),
                   block=w.block, scale=w.scale)


def anchors_per_sample(inp):
    return [inp.anchors_of(s) for s in range(len(inp.workload.seq_lens))]


def read_golden(name):
    out = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, *vals = line.split()
            nums = [int(x) for x in vals]
            out[key] = nums[0] if len(nums) == 1 and key not in ("anchors", "costs", "item_ids") else nums
    return out
