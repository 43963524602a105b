"""Expert-parallel test helpers: host stand-ins for the kernels (built on the
oracle) and a driver that runs several ranks' phases in lockstep from one
process, doing each all-to-all as a copy.  Test infrastructure only."""
from types import SimpleNamespace

import numpy as np
import torch

import oracle
import moe_router_softmax_b200 as moe


def _bits(x: torch.Tensor) -> np.ndarray:
    return x.contiguous().view(torch.int16).numpy().view(np.uint16)


def host_ops():
    """Host versions of the kernels with the binding's signatures (test only)."""

    def route_topk(logits, k):
        ids, w = oracle.route_topk(logits.numpy(), k)
        return torch.from_numpy(ids), torch.from_numpy(w)

    def permute(ids, E, hits=None):
        c, o, s, p = oracle.permute(ids.numpy(), E)
        if hits is not None:
            hits += torch.from_numpy(c.astype(np.int64)).to(hits.dtype)
        return tuple(torch.from_numpy(a) for a in (c, o, s, p))

    def gather_rows(src, index, divisor=1):
        idx = index.long()
        out = torch.zeros((idx.numel(), src.shape[1]), dtype=src.dtype)
        ok = (idx >= 0) & (idx // divisor < src.shape[0])
        out[ok] = src[idx[ok] // divisor]
        return out

    def recv_ids(recv_counts, n):
        N, El = recv_counts.shape
        lab = np.repeat(np.tile(np.arange(El, dtype=np.int32), N), recv_counts.numpy().ravel().clip(0))
        out = np.full(n, -1, np.int32)
        out[:min(n, lab.size)] = lab[:n]
        return torch.from_numpy(out)

    def grouped_ffn(layer, x, k, counts, offsets, sorted_route):
        xb = _bits(x)
        off = offsets.numpy()
        sr = sorted_route.numpy()
        rows = np.zeros((sr.size, layer.H), np.float32)
        for e in range(layer.E):
            for i in range(off[e], off[e + 1]):
                rows[i] = oracle.expert_ffn(layer, e, xb[sr[i] // k]).astype(np.float32)
        return torch.from_numpy(rows)

    def combine(rows, route_pos, w):
        T, k = w.shape
        rp = route_pos.numpy()
        r = np.zeros((T * k, rows.shape[1]), np.float64)
        r[rp >= 0] = rows.numpy()[rp[rp >= 0]].astype(np.float64)
        ids = np.where(rp.reshape(T, k) >= 0, 0, -1).astype(np.int32)
        return torch.from_numpy(oracle.combine(r, ids, w.numpy(), 1))

    return SimpleNamespace(moe_route_topk=route_topk, moe_permute=permute, moe_gather_rows=gather_rows,
                           moe_ep_recv_ids=recv_ids, moe_ep_splits=moe.moe_ep_splits, moe_grouped_ffn=grouped_ffn,
                           moe_combine=combine)


def lockstep(eps, logits, xs, k, hits=None):
    """One layer call of every rank in `eps`, phase by phase; each all-to-all is a
    copy between the ranks' buffers (on whatever device they live)."""
    N, El, H = len(eps), eps[0].El, eps[0].H
    sts = [ep.begin(lg, x, k) for ep, lg, x in zip(eps, logits, xs)]
    for d, st in enumerate(sts):
        st.recv_counts = torch.stack([sts[s].counts.view(N, El)[d] for s in range(N)]).contiguous()
    for ep, st in zip(eps, sts):
        ep.plan(st)
    send_off = [np.concatenate([[0], np.cumsum(st.send_rows)]).astype(int) for st in sts]
    for d, st in enumerate(sts):
        parts = [sts[s].xs[send_off[s][d]:send_off[s][d + 1]] for s in range(N)]
        st.xr = torch.cat(parts).contiguous()
    for d, (ep, st) in enumerate(zip(eps, sts)):
        ep.serve(st, None if hits is None else hits[d])
    recv_off = [np.concatenate([[0], np.cumsum(st.recv_rows)]).astype(int) for st in sts]
    for s, st in enumerate(sts):
        st.rows_back = torch.zeros((max(st.T * k, 1), H), dtype=torch.float32, device=sts[s].xs.device)
        parts = [sts[d].rows_out[recv_off[d][s]:recv_off[d][s + 1]] for d in range(N)]
        n = sum(p.shape[0] for p in parts)
        if n:
            st.rows_back[:n] = torch.cat(parts)
    return [ep.finish(st) for ep, st in zip(eps, sts)], sts
