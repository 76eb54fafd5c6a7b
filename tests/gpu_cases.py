"""Shared plumbing of the GPU parity tests: run one decode step through the C ABI
and compute the same step with the fp64 oracle on the same seeded inputs.

The oracle's inputs are always the generator's values (numpy arrays, or device
tensors that torch's seeded generator filled and that are copied back BEFORE any
library kernel runs); nothing the CUDA path computes is ever fed to the oracle.
"""
import math

import numpy as np
import torch

import oracle
import synth
import paged_kv_cache_460_b200 as pkv

TDT = {"f16": torch.float16, "bf16": torch.bfloat16}
ATOL, RTOL = 1e-3, 1e-2          # |gpu - ref| <= 1e-3 + 1e-2 |ref|


def to_dev(bits, dtype):
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16).copy())
    return t.view(TDT[dtype]).cuda()


def to_bits(t):
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def tolerance_report(gpu_bits, ref, dtype):
    """(all within tolerance, max abs error, max error / bound)."""
    g = oracle.decode(gpu_bits, dtype)
    err = np.abs(g - ref)
    bound = ATOL + RTOL * np.abs(ref)
    finite = np.isfinite(g).all()
    return bool(finite and (err <= bound).all()), float(err.max(initial=0.0)), float((err / bound).max(initial=0.0))


class Case:
    """Device state of one workload: pools, page tables, per-layer q/k/v."""

    def __init__(self, spec, pool_backend="numpy"):
        self.s = s = spec
        self.q, self.k, self.v = synth.step_values(s)            # uint16 [layers, B, H, d]
        if pool_backend == "numpy":
            self.kp, self.vp = synth.pool_values_numpy(s)          # uint16 [layers, pages, Hkv, P, d]
            self.kp_t, self.vp_t = to_dev(self.kp, s.dtype), to_dev(self.vp, s.dtype)
        else:
            self.kp = self.vp = None
            self.kp_t, self.vp_t = synth.pool_values_torch(s, "cuda")
        self.pool = pkv.KVPool(self.kp_t, self.vp_t)
        self.bt_t = torch.from_numpy(s.block_tables).cuda()
        self.cl_t = torch.from_numpy(s.context_lens).cuda()
        self.pos_t = torch.from_numpy(s.positions).cuda()
        self.slots = pkv.pkv_slot_mapping(s.block_tables, s.positions, s.page_size)
        self.slots_t = torch.from_numpy(self.slots).cuda()
        self.scale = 1.0 / math.sqrt(s.head_dim)

    def gpu_layer(self, layer, num_splits=0, workspace=None, fused=False):
        s = self.s
        q_t = to_dev(self.q[layer], s.dtype)
        k_t = to_dev(self.k[layer], s.dtype)
        v_t = to_dev(self.v[layer], s.dtype)
        if fused:
            pkv.rope_append(self.pool, layer, q_t, k_t, v_t, self.pos_t, self.slots_t, s.theta)
        else:
            pkv.rope_apply(q_t, k_t, self.pos_t, s.theta)
            pkv.paged_kv_append(self.pool, layer, k_t, v_t, self.slots_t)
        self.last_q = q_t
        out = torch.empty_like(q_t)
        pkv.paged_decode_attention(self.pool, layer, out, q_t, self.bt_t, self.cl_t, self.scale,
                                   num_splits=num_splits, workspace=workspace)
        return out

    def oracle_layer(self, layer):
        """Whole-batch oracle step (numpy pools only)."""
        s = self.s
        q_rot, _ = oracle.rope(self.q[layer], s.positions, s.theta, s.dtype)
        k_rot, _ = oracle.rope(self.k[layer], s.positions, s.theta, s.dtype)
        kp2, vp2 = oracle.kv_append(self.kp[layer], self.vp[layer], k_rot, self.v[layer], s.block_tables,
                                    s.positions)
        return oracle.decode_attention(q_rot, kp2, vp2, s.block_tables, s.context_lens, self.scale, s.dtype)

    def snapshot_pairs(self, layer, pairs):
        """Copy the pages of each sampled (b, kv head) off the device, before any
        library kernel touches this layer.  Returns per-pair mini pools."""
        s = self.s
        snaps = []
        for b, g in pairs:
            np_b = (int(s.context_lens[b]) + s.page_size - 1) // s.page_size
            pages = torch.from_numpy(s.block_tables[b, :np_b].astype(np.int64)).cuda()
            kmini = to_bits(self.kp_t[layer].index_select(0, pages)[:, g:g + 1])
            vmini = to_bits(self.vp_t[layer].index_select(0, pages)[:, g:g + 1])
            snaps.append((b, g, kmini, vmini))
        return snaps

    def oracle_pairs(self, layer, snaps):
        """Oracle output of the G query heads of each snapshotted (b, kv head): [n, G, d]."""
        s = self.s
        G = s.q_heads // s.kv_heads
        q_rot, _ = oracle.rope(self.q[layer], s.positions, s.theta, s.dtype)
        k_rot, _ = oracle.rope(self.k[layer], s.positions, s.theta, s.dtype)
        outs = []
        for b, g, kmini, vmini in snaps:
            np_b = kmini.shape[0]
            table = np.arange(np_b, dtype=np.int32)[None, :]
            pos = np.array([s.positions[b]], np.int32)
            kp2, vp2 = oracle.kv_append(kmini, vmini, k_rot[b:b + 1, g:g + 1], self.v[layer][b:b + 1, g:g + 1],
                                        table, pos)
            o = oracle.decode_attention(q_rot[b:b + 1, g * G:(g + 1) * G], kp2, vp2, table,
                                        np.array([s.context_lens[b]], np.int32), self.scale, s.dtype)
            outs.append(o[0])
        return np.stack(outs)
