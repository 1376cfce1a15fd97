"""Host-side plumbing around the C ABI: parameter structs from a workload
description, device buffers for the lists (allocated with torch), and the
retained-pair count the throughput metric needs.  No attention or selector
arithmetic happens here."""
import math

import torch

from . import api
from ._lib import (STA_ATTN_LISTS, STA_ATTN_ROUTED, STA_BF16, STA_F32, STA_SEL_ENTROPY,
                   STA_SEL_DYNRAD, STA_SEL_IBCS_SIP, STA_SEL_RADIAL, STA_SEL_ROUTED,
                   STA_SEL_TRA_TOKEN, AttnParams, BlockLists, Problem, SelectorParams)

_KINDS = {"radial": STA_SEL_RADIAL, "entropy": STA_SEL_ENTROPY, "ibcs_sip": STA_SEL_IBCS_SIP,
          "routed": STA_SEL_ROUTED, "tra_token": STA_SEL_TRA_TOKEN, "dynrad": STA_SEL_DYNRAD}


def problem(w):
    return Problem(w["heads"], w["F"], w["H"], w["W"], w["d"],
                   STA_F32 if w["dtype"] == "f32" else STA_BF16)


def selector(w, difficulty=None, entropy=None):
    s = SelectorParams()
    s.kind = _KINDS[w["selector"]]
    s.block_q = w["block_q"]
    s.kv_unit = w["kv_unit"]
    if w["selector"] in ("radial", "dynrad"):
        r = w["radial"]
        s.radial_w0, s.radial_w_off, s.radial_full_df = r["w0"], r["w_off"], r["full_df"]
    if w["selector"] == "dynrad":
        c = w["dynrad"]
        s.dyn_mode = 0 if c["mode"] == "static" else 1
        s.dyn_ratio, s.dyn_threshold = c.get("ratio", 0.0), c.get("threshold", 0.0)
    elif w["selector"] == "entropy":
        e = w["entropy"]
        s.ent_alpha, s.ent_beta = e["alpha"], e["beta"]
        s.ent_r_lo, s.ent_r_hi = e["r_lo"], e["r_hi"]
        s.ent_tile_h, s.ent_tile_w = e["tile_h"], e["tile_w"]
    elif w["selector"] == "ibcs_sip":
        c = w["ibcs"]
        s.km_k, s.km_iters, s.sample_frac, s.seed = c["k"], c["iters"], c["sample_frac"], c["seed"]
    elif w["selector"] == "routed":
        c = w["routed"]
        s.dense_frac, s.win_f, s.win_h, s.win_w = c["dense_frac"], c["win_f"], c["win_h"], c["win_w"]
        if difficulty is not None:
            s.difficulty = api._ptr(difficulty)
    elif w["selector"] == "tra_token":
        c = w["tra_token"]
        s.tra_tau, s.tra_gamma, s.tra_vote = c["tau"], c["gamma"], c["vote"]
        if w.get("layout"):
            s.layout_tile_h, s.layout_tile_w = w["layout"]
        if entropy is not None:
            s.tra_entropy = api._ptr(entropy)
    return s


def selector_workspace(w, device="cuda"):
    """Device scratch of sta_build_blocks for this workload (None if none)."""
    n = api.sta_build_blocks_workspace(problem(w), selector(w))
    if n == 0:
        return None
    return torch.empty(n, dtype=torch.uint8, device=device)


def route_count(w):
    """Tokens on the dense path: ceil(frac * N) with the library's 1e-6 slack."""
    N = w["F"] * w["H"] * w["W"]
    m = math.ceil(float(torch.tensor(w["routed"]["dense_frac"], dtype=torch.float32)) * N
                  * (1.0 - 1e-6))
    return max(0, min(N, m))


def retained_pairs_routed(w, routed_flag):
    """Algorithmic kept (query, key) pairs of the routed workload over all
    heads: N keys for every routed token plus, for every other token, the
    number of keys inside its clipped local window.  routed_flag: [N] bool
    or uint8 (host or device)."""
    F, H, W = w["F"], w["H"], w["W"]
    N = F * H * W
    c = w["routed"]
    flag = routed_flag.detach().cpu().bool()
    t = torch.arange(N, dtype=torch.int64)
    S = H * W
    f, h, x = t // S, (t % S) // W, t % W
    nf = torch.clamp(f + c["win_f"], max=F - 1) - torch.clamp(f - c["win_f"], min=0) + 1
    nh = torch.clamp(h + c["win_h"], max=H) - torch.clamp(h - c["win_h"], min=0)
    nw = torch.clamp(x + c["win_w"], max=W) - torch.clamp(x - c["win_w"], min=0)
    local = int((nf * nh * nw)[~flag].sum().item())
    return w["heads"] * (int(flag.sum().item()) * N + local)


def attn_params(w):
    p = AttnParams()
    p.mode = STA_ATTN_ROUTED if w["selector"] == "routed" else STA_ATTN_LISTS
    p.block_q = w["block_q"]
    p.kv_unit = w["kv_unit"]
    p.scale = 0.0
    if w["selector"] == "routed":
        c = w["routed"]
        p.win_f, p.win_h, p.win_w = c["win_f"], c["win_h"], c["win_w"]
    return p


def default_cap(w):
    N = w["F"] * w["H"] * w["W"]
    n_units = (N + w["kv_unit"] - 1) // w["kv_unit"]
    if w["selector"] == "ibcs_sip":
        m = math.ceil(w["ibcs"]["sample_frac"] * n_units)
        return min(n_units, m + int(10 * math.sqrt(m)) + 64)
    if w["selector"] == "routed":
        return min(n_units, 1024)
    return n_units


class Lists:
    """Device buffers of one sta_block_lists, sized for a workload."""

    def __init__(self, w, device="cuda", cap=None):
        self.w = w
        prob, sel = problem(w), selector(w)
        self.rows = api.sta_build_blocks_rows(prob, sel)
        if self.rows < 0:
            raise ValueError("unsupported selector/problem")
        self.cap = cap or default_cap(w)
        N = w["F"] * w["H"] * w["W"]
        z = dict(device=device)
        self.idx = torch.zeros(self.rows, self.cap, dtype=torch.int32, **z)
        self.cnt = torch.zeros(self.rows, dtype=torch.int32, **z)
        self.required_cap = torch.zeros(1, dtype=torch.int32, **z)
        self.logw = (torch.zeros(self.rows, self.cap, dtype=torch.float32, **z)
                     if w["selector"] == "ibcs_sip" else None)
        nqb = (N + w["block_q"] - 1) // w["block_q"]
        if w["selector"] == "routed":
            self.routed_ids = torch.zeros(N, dtype=torch.int32, **z)
            self.routed_flag = torch.zeros(N, dtype=torch.uint8, **z)
        else:
            self.routed_ids = self.routed_flag = None
        if w["selector"] == "entropy":
            self.entropy = torch.zeros(w["heads"], nqb, dtype=torch.float32, **z)
            self.radius = torch.zeros(w["heads"], nqb, dtype=torch.int32, **z)
        else:
            self.entropy = self.radius = None
        self.struct = BlockLists()
        s = self.struct
        s.idx, s.cnt, s.cap = self.idx.data_ptr(), self.cnt.data_ptr(), self.cap
        s.logw = self.logw.data_ptr() if self.logw is not None else None
        s.required_cap = self.required_cap.data_ptr()
        s.head_shared = 1 if self.rows == nqb else 0
        if self.routed_ids is not None:
            s.routed_ids = self.routed_ids.data_ptr()
            s.routed_flag = self.routed_flag.data_ptr()
        if self.entropy is not None:
            s.entropy = self.entropy.data_ptr()
            s.radius = self.radius.data_ptr()

    def host_rows(self):
        """Lists as Python lists of ascending unit ids (host copy)."""
        idx = self.idx.cpu()
        cnt = self.cnt.cpu()
        return [idx[r, :int(cnt[r])].tolist() for r in range(self.rows)]


def retained_pairs(w, lists: Lists, routed_ids=None):
    """Kept (query, key) pairs over all heads, true block and unit lengths
    (padding, masked tails and out-of-window keys excluded).  Used for the
    effective-TFLOP/s metric (4*d FLOPs per kept pair)."""
    N = w["F"] * w["H"] * w["W"]
    B, U, heads = w["block_q"], w["kv_unit"], w["heads"]
    nqb = (N + B - 1) // B
    cnt = lists.cnt.cpu().long()
    idx = lists.idx.cpu().long()
    total = 0
    unit_len = torch.clamp(N - torch.arange((N + U - 1) // U) * U, max=U)
    for r in range(lists.rows):
        c = int(cnt[r])
        keys = int(unit_len[idx[r, :c]].sum())
        qb = r % nqb
        qlen = min(B, N - qb * B)
        total += qlen * keys
    if lists.rows == nqb:
        total *= heads
    return total
