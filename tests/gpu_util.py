"""Helpers of the GPU parity tests: move oracle-side stage inputs into the
library's buffer layout, and decode library outputs for comparison.  Every
input handed to the CUDA path here comes from the seeded generators or the
oracle; nothing the CUDA path computes is fed back into the oracle."""
import numpy as np
import pytest
import torch


def need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def B():
    from gaussian_splatting_differentiable_dgs_b200 import binding
    return binding


def encode_records(rec_c):
    """Oracle fp64 candidate records [C][16] -> library fp32 records [C][12]."""
    rec_c = np.asarray(rec_c, np.float64)
    C = len(rec_c)
    out = np.zeros((C, 12), np.float32)
    u, v = rec_c[:, 0], rec_c[:, 1]
    uh, vh = u.astype(np.float32), v.astype(np.float32)
    out[:, 0], out[:, 1] = uh, vh
    lo = np.stack([u - uh.astype(np.float64), v - vh.astype(np.float64)], 1).astype(np.float16)
    out[:, 2] = lo.view(np.float32).reshape(-1)
    # alpha box half extents (the library's bound), fp16 rounded up
    lq = np.log(255.0 * rec_c[:, 7])
    qb = np.maximum(lq, 0.0) * 1.0001 + 1e-4
    hx = (np.sqrt(2 * qb * rec_c[:, 11]) + 0.01).astype(np.float32)
    hy = (np.sqrt(2 * qb * rec_c[:, 13]) + 0.01).astype(np.float32)
    box = np.stack([_half_up(hx), _half_up(hy)], 1)
    out[:, 3] = box.view(np.float32).reshape(-1)
    a, b = rec_c[:, 4], rec_c[:, 5]
    S11 = rec_c[:, 13]
    out[:, 4] = (0.5 * a).astype(np.float32)
    out[:, 5] = (b / a).astype(np.float32)
    out[:, 6] = (0.5 / S11).astype(np.float32)
    out[:, 7] = rec_c[:, 7].astype(np.float32)
    out[:, 8:11] = rec_c[:, 8:11].astype(np.float32)
    out[:, 11] = rec_c[:, 2].astype(np.float32)
    return out


def _half_up(x):
    """fp32 -> fp16 rounded towards +inf."""
    h = np.asarray(x, np.float32).astype(np.float16)
    low = h.astype(np.float32) < x
    h[low] = np.nextafter(h[low], np.float16(np.inf))
    return h


def decode_records(rec12):
    """Library records [C][12] -> dict of fp64 fields (conic reconstructed)."""
    raw = np.asarray(rec12, np.float32).reshape(-1, 12)
    r = raw.astype(np.float64)
    lo = np.ascontiguousarray(raw[:, 2]).view(np.float16).reshape(-1, 2).astype(np.float64)
    box = np.ascontiguousarray(raw[:, 3]).view(np.float16).reshape(-1, 2).astype(np.float64)
    s1, beta, s2 = r[:, 4], r[:, 5], r[:, 6]
    a = 2 * s1
    b = beta * a
    c = 2 * s2 + beta * beta * a
    return dict(u=r[:, 0] + lo[:, 0], v=r[:, 1] + lo[:, 1], a=a, b=b, c=c, s1=s1, beta=beta,
                s2=s2, opac=r[:, 7], rgb=r[:, 8:11], depth=r[:, 11], hx=box[:, 0], hy=box[:, 1])


class ProjBuffers:
    """Device buffers of a gs_proj (capacity cap) plus the struct."""

    def __init__(self, cap, dev="cuda"):
        cap = max(int(cap), 1)
        self.cap = cap
        self.n_cand = torch.zeros(1, dtype=torch.int32, device=dev)
        self.cand_idx = torch.zeros(cap, dtype=torch.int32, device=dev)
        self.slot = torch.full((cap,), -1, dtype=torch.int32, device=dev)
        self.rec = torch.zeros(cap * 12, dtype=torch.float32, device=dev)
        self.rect = torch.zeros(cap * 4, dtype=torch.int16, device=dev)
        self.depth_key = torch.zeros(cap, dtype=torch.int32, device=dev)
        self.square = torch.zeros(1, dtype=torch.int64, device=dev)
        b = B()
        self.struct = b.gs_proj(cap, self.n_cand.data_ptr(), self.cand_idx.data_ptr(),
                                self.slot.data_ptr(), self.rec.data_ptr(), self.rect.data_ptr(),
                                self.depth_key.data_ptr(), self.square.data_ptr())

    @classmethod
    def from_oracle(cls, pr, n):
        """Candidate state written from the oracle's projection."""
        C = len(pr["cand_idx"])
        pb = cls(max(n, C))
        pb.n_cand.fill_(C)
        if C:
            pb.cand_idx[:C] = torch.as_tensor(pr["cand_idx"])
            pb.rec[:C * 12] = torch.as_tensor(encode_records(pr["rec"]).reshape(-1))
            pb.rect[:C * 4] = torch.as_tensor(pr["rect"].astype(np.int16).reshape(-1))
            pb.depth_key[:C] = torch.as_tensor(pr["key"].view(np.int32))
        slot = np.full(max(n, 1), -1, np.int32)
        slot[pr["cand_idx"]] = np.arange(C, dtype=np.int32)
        pb.slot[:len(slot)] = torch.as_tensor(slot)
        return pb


def rel_err(got, ref, floor=1e-3):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    return np.abs(got - ref) / np.maximum(np.abs(ref), floor)


def rel_l2(got, ref):
    got = np.asarray(got, np.float64).ravel()
    ref = np.asarray(ref, np.float64).ravel()
    nr = np.linalg.norm(ref)
    return np.linalg.norm(got - ref) / (nr if nr > 0 else 1.0)
