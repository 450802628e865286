"""A CPU stand-in for the compute of the head-sharded path, built on the fp64
oracle -- TEST INFRASTRUCTURE. It lets the host logic of
`block_sparse_attention_fvattn_b200.heads` (plans, slot moves, point-to-point
exchanges over gloo, output reassembly) run on CPU processes; the product
path uses the library's kernels (heads.GpuBackend) and never this module.
"""
import math

import numpy as np
import torch


class OracleBackend:
    def __init__(self, wl, orc):
        self.wl, self.orc = wl, orc
        self.nb = orc.num_blocks(orc.geom(1, 1, wl.grid, wl.block, wl.D))
        self.scale = 1.0 / math.sqrt(wl.D)
        self.sizes = orc.block_sizes(orc.geom(1, 1, wl.grid, wl.block, wl.D)).astype(np.int64)

    def g(self, F):
        return self.orc.geom(1, F, self.wl.grid, self.wl.block, self.wl.D)

    def alloc(self, slots):
        N, D, nb = self.wl.N, self.wl.D, self.nb
        return dict(q=torch.zeros(slots, N, D, dtype=torch.bfloat16), k=torch.zeros(slots, N, D, dtype=torch.bfloat16),
                    v=torch.zeros(slots, N, D, dtype=torch.bfloat16), o=torch.zeros(slots, N, D, dtype=torch.bfloat16),
                    cnt=torch.zeros(slots, nb, dtype=torch.int32), idx=torch.zeros(slots, nb, nb, dtype=torch.int32),
                    probs=torch.zeros(slots, nb, nb, dtype=torch.float64))

    def route(self, buf, a, b):
        F = b - a
        if F <= 0:
            return
        g = self.g(F)
        qb, kb = self.orc.pool(g, buf["q"][a:b].unsqueeze(0)), self.orc.pool(g, buf["k"][a:b].unsqueeze(0))
        r = self.orc.route(g, qb, kb, self.scale, self.wl.p, self.wl.k_min)
        buf["cnt"][a:b] = torch.from_numpy(r["kv_cnt"][0])
        buf["idx"][a:b] = torch.from_numpy(r["kv_idx"][0])
        buf["probs"][a:b] = torch.from_numpy(r["probs"][0])

    def head_cost(self, buf, F):
        out = []
        for s in range(F):
            c = buf["cnt"][s].numpy()
            ix = buf["idx"][s].numpy()
            tot = 0
            for i in range(self.nb):
                tot += int(self.sizes[i]) * int(self.sizes[ix[i, :c[i]]].sum())
            out.append(tot)
        return torch.tensor(out, dtype=torch.int64)

    def augment(self, buf, F, budget):
        if F <= 0:
            return torch.zeros(1, dtype=torch.int64), torch.zeros(1, dtype=torch.float64)
        cnt, idx, added, mass = self.orc.augment(self.g(F), buf["probs"][:F].numpy(), int(budget),
                                                 buf["cnt"][:F].numpy(), buf["idx"][:F].numpy())
        buf["cnt"][:F] = torch.from_numpy(cnt)
        buf["idx"][:F] = torch.from_numpy(idx)
        return torch.tensor([added], dtype=torch.int64), torch.tensor([mass], dtype=torch.float64)

    def attend(self, buf, F):
        if F <= 0:
            return
        N, D = self.wl.N, self.wl.D
        out, _ = self.orc.attn_rows(self.g(F), buf["q"][:F].unsqueeze(0), buf["k"][:F].unsqueeze(0),
                                    buf["v"][:F].unsqueeze(0), self.scale, np.arange(F * N),
                                    buf["cnt"][:F].numpy()[None], buf["idx"][:F].numpy()[None])
        buf["o"][:F] = torch.from_numpy(out.reshape(F, N, D)).to(torch.bfloat16)

    def copy_slot(self, buf, src, dst, names=("q", "k", "v", "cnt", "idx", "probs")):
        for n in names:
            buf[n][dst].copy_(buf[n][src])
