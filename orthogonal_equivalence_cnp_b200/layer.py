"""Device buffers of one POET-X layer and the call sequence of one training step.

Plumbing only: torch provides device memory and the stream; every step of the layer runs in
libpoetx's kernels through the C ABI (see the package __init__).
"""
from __future__ import annotations

import numpy as np
import torch

from . import (POETX_BF16, POETX_F32, POETX_FAST, POETX_MEM, poetx_absorb, poetx_adamw_cfg, poetx_adamw_reset,
               poetx_adamw_step, poetx_backward, poetx_cnp, poetx_cnp_forward, poetx_desc, poetx_fourperm_backward,
               poetx_fourperm_forward, poetx_fourperm_workspace_size, poetx_forward,
               poetx_merge, poetx_wc_backward, poetx_wc_forward, poetx_wc_saved_size, poetx_wc_workspace_size,
               poetx_workspace_size, poetx_xq_backward, poetx_xq_forward, poetx_xq_merge, poetx_xq_quantize)

TORCH_DTYPE = {POETX_F32: torch.float32, POETX_BF16: torch.bfloat16}


def make_desc(d_in: int, d_out: int, b: int, k: int, dtype: str, mode: str) -> poetx_desc:
    return poetx_desc(d_in, d_out, b, k, POETX_BF16 if dtype == "bf16" else POETX_F32,
                      POETX_MEM if mode == "mem" else POETX_FAST)


class PoetxLayer:
    """Holds W0', theta, permutations, Q and scratch of one layer on one device."""

    def __init__(self, desc: poetx_desc, n_tokens: int, device="cuda"):
        self.desc = desc
        self.n = int(n_tokens)
        self.device = torch.device(device)
        dt = TORCH_DTYPE[desc.dtype]
        self.dtype = dt
        b, din, dout = desc.b, desc.d_in, desc.d_out
        P = b * (b - 1) // 2
        dev = self.device
        self.W0p = torch.empty(dout, din, dtype=dt, device=dev)
        # POET-XQ (after quantize()): W0' as int8 codes W0q [d_out, d_in] and scales W0s [d_out].
        self.xq = False
        self.W0q = self.W0s = None
        # theta_R and theta_P (and their gradients and AdamW moments) are stored back to back so
        # that one optimiser launch covers both sides.
        nbo, nbi = dout // b, din // b
        self.theta = torch.zeros(nbo + nbi, P, dtype=torch.float32, device=dev)
        self.theta_R, self.theta_P = self.theta[:nbo], self.theta[nbo:]
        self.perm_L = torch.arange(dout, dtype=torch.int32, device=dev)
        self.perm_R = torch.arange(din, dtype=torch.int32, device=dev)
        self.Q_R = torch.empty(dout // b, b, b, dtype=dt, device=dev)
        self.Q_P = torch.empty(din // b, b, b, dtype=dt, device=dev)
        self.Y = torch.empty(self.n, dout, dtype=dt, device=dev)
        # POET-Xfast keeps Z [N, d_out] and U = X[:, pi_R] [N, d_in] for the backward pass.
        self.saved = torch.empty(self.n * (dout + din), dtype=dt, device=dev) if desc.mode == POETX_FAST else None
        self.dX = torch.empty(self.n, din, dtype=dt, device=dev)
        self.grad = torch.zeros_like(self.theta)
        self.g_R, self.g_P = self.grad[:nbo], self.grad[nbo:]
        self.m = torch.zeros_like(self.theta)
        self.v = torch.zeros_like(self.theta)
        self.t = 0       # AdamW step count of the current moments
        self.steps = 0   # training steps taken (drives the merge schedule)
        ws = poetx_workspace_size(desc, self.n)
        self.ws = torch.empty(max(ws, 256), dtype=torch.uint8, device=dev)

    # ------------------------------------------------------------------ state upload helpers
    def to_dev(self, a: np.ndarray, dtype=None) -> torch.Tensor:
        t = torch.from_numpy(np.ascontiguousarray(a))
        return t.to(device=self.device, dtype=dtype or self.dtype)

    def load_state(self, W0: np.ndarray, theta_R, theta_P, pi_L, pi_R):
        """Uploads the original-basis W0 and absorbs the two permutations on the device."""
        self.perm_L.copy_(torch.from_numpy(np.asarray(pi_L, np.int32)))
        self.perm_R.copy_(torch.from_numpy(np.asarray(pi_R, np.int32)))
        self.theta_R.copy_(torch.from_numpy(np.asarray(theta_R, np.float32)))
        self.theta_P.copy_(torch.from_numpy(np.asarray(theta_P, np.float32)))
        W0_dev = self.to_dev(W0)
        poetx_absorb(self.desc, W0_dev, self.perm_L, self.perm_R, self.W0p)
        self.W0 = W0_dev  # the un-absorbed weight, kept for the four-permutation comparator

    # ------------------------------------------------------------------------- the step
    def cnp(self):
        poetx_cnp(self.desc, self.theta_R, self.theta_P, self.Q_R, self.Q_P, self.ws)

    def forward(self, X: torch.Tensor):
        if self.xq:
            poetx_xq_forward(self.desc, self.n, X, self.W0q, self.W0s, self.perm_L, self.perm_R, self.Q_R, self.Q_P,
                             self.Y, self.ws)
        else:
            poetx_forward(self.desc, self.n, X, self.W0p, self.perm_L, self.perm_R, self.Q_R, self.Q_P, self.Y,
                          self.saved, self.ws)
        return self.Y

    def backward(self, dY: torch.Tensor, X: torch.Tensor):
        if self.xq:
            poetx_xq_backward(self.desc, self.n, dY, X, self.W0q, self.W0s, self.perm_L, self.perm_R, self.Q_R,
                              self.Q_P, self.theta_R, self.theta_P, self.dX, self.g_R, self.g_P, self.ws)
        else:
            poetx_backward(self.desc, self.n, dY, X, self.W0p, self.perm_L, self.perm_R, self.Q_R, self.Q_P,
                           self.theta_R, self.theta_P, self.saved, self.dX, self.g_R, self.g_P, self.ws)
        return self.dX, self.g_R, self.g_P

    def quantize(self):
        """Switches the layer to POET-XQ (mem mode, bf16): W0' becomes int8 codes with one scale
        per row, and the bf16 W0' is released."""
        d = self.desc
        self.W0q = torch.empty(d.d_out, d.d_in, dtype=torch.int8, device=self.device)
        self.W0s = torch.empty(d.d_out, dtype=torch.float32, device=self.device)
        poetx_xq_quantize(d, self.W0p, self.W0q, self.W0s)
        self.W0p = None  # stream-ordered release: the quantiser has been enqueued before it
        self.xq = True

    def cnp_forward(self, X: torch.Tensor):
        """CNP and layer forward in one library call (the CNP overlaps the input gather)."""
        poetx_cnp_forward(self.desc, self.n, X, self.W0p, self.perm_L, self.perm_R, self.theta_R, self.theta_P,
                          self.Q_R, self.Q_P, self.Y, self.saved, self.ws)
        return self.Y

    def step(self, X: torch.Tensor, dY: torch.Tensor, grad_ready=None):
        """CNP forward + layer forward + layer backward (incl. the CNP adjoint).  grad_ready (for
        data parallelism, e.g. GradBuckets.layer_done of this layer) is called once the backward
        pass, which writes the packed gradients, has been enqueued."""
        if self.xq:
            self.cnp()
            self.forward(X)
        else:
            self.cnp_forward(X)
        self.backward(dY, X)
        if grad_ready is not None:
            grad_ready()

    def optimizer_step(self, cfg: poetx_adamw_cfg):
        """AdamW on the packed theta (both sides in one launch)."""
        self.t += 1
        poetx_adamw_step(cfg, self.theta.numel(), self.t, self.theta, self.grad, self.m, self.v)

    def train_step(self, X: torch.Tensor, dY: torch.Tensor, cfg: poetx_adamw_cfg, reset_gap: int = 400,
                   new_perms=None):
        """One training step with the merge schedule: CNP, forward, backward, AdamW; after every
        reset_gap steps merge-then-reinitialise with the permutations new_perms() returns
        (host int32 arrays pi_L, pi_R) and restart the moments."""
        self.step(X, dY)
        self.optimizer_step(cfg)
        self.steps += 1
        if reset_gap and self.steps % reset_gap == 0:
            if new_perms is None:
                raise ValueError("the merge schedule needs new permutations")
            pL, pR = new_perms()
            self.cnp()  # Q of the theta being folded in
            self.merge(torch.from_numpy(np.asarray(pL, np.int32)).to(self.device),
                       torch.from_numpy(np.asarray(pR, np.int32)).to(self.device))
            poetx_adamw_reset(self.m.numel(), self.m, self.v)
            self.t = 0

    def fourperm_step(self, X: torch.Tensor, dY: torch.Tensor):
        """The same step with none of the permutations absorbed (comparator): R and P applied around
        the original W0, four activation permutations per pass.  Same outputs as step()."""
        if getattr(self, "fp_saved", None) is None:
            self.fp_saved = torch.empty(self.n * (self.desc.d_in + self.desc.d_out), dtype=self.dtype,
                                        device=self.device)
            self.fp_ws = torch.empty(max(poetx_fourperm_workspace_size(self.desc, self.n), 256), dtype=torch.uint8,
                                     device=self.device)
        poetx_cnp(self.desc, self.theta_R, self.theta_P, self.Q_R, self.Q_P, self.fp_ws)
        poetx_fourperm_forward(self.desc, self.n, X, self.W0, self.perm_L, self.perm_R, self.Q_R, self.Q_P, self.Y,
                               self.fp_saved, self.fp_ws)
        poetx_fourperm_backward(self.desc, self.n, dY, self.W0, self.perm_L, self.perm_R, self.Q_R, self.Q_P,
                                self.theta_R, self.theta_P, self.fp_saved, self.dX, self.g_R, self.g_P, self.fp_ws)

    def wc_step(self, X: torch.Tensor, dY: torch.Tensor):
        """The same step in the weight-centric order (comparator): CNP, form W = R W0 P, Y = X W^T,
        dX = dY W, dW = dY^T X and the gradients of theta from dW.  Same outputs as step()."""
        if getattr(self, "wc_saved", None) is None:
            self.wc_saved = torch.empty(poetx_wc_saved_size(self.desc), dtype=torch.uint8, device=self.device)
            self.wc_ws = torch.empty(max(poetx_wc_workspace_size(self.desc), 256), dtype=torch.uint8,
                                     device=self.device)
        poetx_cnp(self.desc, self.theta_R, self.theta_P, self.Q_R, self.Q_P, self.wc_ws)
        poetx_wc_forward(self.desc, self.n, X, self.W0p, self.perm_L, self.perm_R, self.Q_R, self.Q_P, self.Y,
                         self.wc_saved, self.wc_ws)
        poetx_wc_backward(self.desc, self.n, dY, X, self.W0p, self.perm_L, self.perm_R, self.Q_R, self.theta_R,
                          self.theta_P, self.wc_saved, self.dX, self.g_R, self.g_P, self.wc_ws)

    def merge(self, pi_L_new: torch.Tensor, pi_R_new: torch.Tensor):
        """Folds R and P into W0', absorbs the new permutations and resets theta (Q must be current)."""
        if self.xq:
            poetx_xq_merge(self.desc, self.W0q, self.W0s, self.Q_R, self.Q_P, self.perm_L, self.perm_R, pi_L_new,
                           pi_R_new, self.theta_R, self.theta_P, self.ws)
        else:
            poetx_merge(self.desc, self.W0p, self.Q_R, self.Q_P, self.perm_L, self.perm_R, pi_L_new, pi_R_new,
                        self.theta_R, self.theta_P, self.ws)
        self.perm_L.copy_(pi_L_new)
        self.perm_R.copy_(pi_R_new)
