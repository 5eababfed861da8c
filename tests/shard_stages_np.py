"""A NumPy stand-in for the library's staged selection (tests only).

It follows the selection rule the library documents for heads split over ranks:
the fp32 scores' bit patterns ordered as unsigned integers, the k-th largest
off-diagonal key of a sequence found one digit at a time (digits of 11, 11 and
10 bits, most significant first) from histograms summed over ranks, then keys
above that threshold kept, and threshold ties taken in flat order (ranks in head
order, then query-block row, then key block).  It lets the multi-rank host logic
run on CPU with gloo; the GPU tests check the library's kernels themselves.
"""
import math

import numpy as np
import torch

DIGITS = ((21, 11), (10, 11), (0, 10))  # (shift, width), most significant first
NBINS = 2048
NONE = 0xFFFFFFFF  # threshold when there are no free picks


class NumpyStages:
    def __init__(self, scores, sparsity: float, heads_total: int):
        self.scores = np.ascontiguousarray(scores, dtype=np.float32)
        self.keys = self.scores.view(np.uint32)
        B, H, nb, _ = self.scores.shape
        self.B, self.H, self.nb = B, H, nb
        kb = math.floor((1.0 - sparsity) * heads_total * nb * nb + 0.5)
        self.kfree = kb - heads_total * nb
        assert self.kfree >= 0
        self.offdiag = ~np.eye(nb, dtype=bool)
        self.h = torch.zeros((len(DIGITS), B, NBINS), dtype=torch.int32)

    def _resolve(self, b: int, npass: int):
        """Digit prefix of the k-th largest key and how many keys with that prefix
        are still to be taken, from the (summed) histograms of the first npass passes."""
        prefix, krem = 0, self.kfree
        for p in range(npass):
            shift, width = DIGITS[p]
            counts = self.h[p, b].numpy()
            above = 0
            for d in range((1 << width) - 1, -1, -1):
                c = int(counts[d])
                if above < krem <= above + c:
                    prefix |= d << shift
                    krem -= above
                    break
                above += c
        return prefix, krem

    def hist_pass(self, p: int):
        shift, width = DIGITS[p]
        hs = shift + width
        for b in range(self.B):
            self.h[p, b] = 0
            if self.kfree == 0:
                continue
            prefix, _ = self._resolve(b, p)
            k = self.keys[b][:, self.offdiag]  # [H, nb*(nb-1)]
            if hs < 32:
                k = k[(k >> np.uint32(hs)) == np.uint32(prefix >> hs)]
            digit = (k.astype(np.int64) >> shift) & ((1 << width) - 1)
            self.h[p, b] = torch.from_numpy(np.bincount(digit.ravel(), minlength=NBINS)[:NBINS]
                                            .astype(np.int32))

    def hist(self, p: int):
        return self.h[p]

    def _tau(self, b: int) -> int:
        return NONE if self.kfree == 0 else self._resolve(b, len(DIGITS))[0]

    def count(self):
        out = torch.zeros((self.B, 2), dtype=torch.int64)
        for b in range(self.B):
            tau = self._tau(b)
            k = self.keys[b][:, self.offdiag]
            out[b, 0] = int((k > np.uint32(tau)).sum()) if tau != NONE else 0
            out[b, 1] = int((k == np.uint32(tau)).sum())
        return out

    def finish(self, offsets, row_ptr=None, col_idx=None, want_mask: bool = False):
        B, H, nb = self.B, self.H, self.nb
        mask = np.zeros((B, H, nb, nb), dtype=np.uint8)
        for b in range(B):
            tau = self._tau(b)
            ties_left = int(self.kfree - int(offsets[b, 0]) - int(offsets[b, 1]))
            for h in range(H):
                for i in range(nb):
                    for j in range(nb):
                        key = int(self.keys[b, h, i, j])
                        if i == j or (tau != NONE and key > tau):
                            mask[b, h, i, j] = 1
                        elif key == tau and ties_left > 0:
                            mask[b, h, i, j] = 1
                            ties_left -= 1
        counts = mask.reshape(-1, nb).sum(1)
        rp = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
        ci = np.nonzero(mask.reshape(-1, nb))[1].astype(np.int32)
        return torch.from_numpy(rp), torch.from_numpy(ci), torch.from_numpy(mask)
