"""CPU fp64 oracle for paged-KV attention (TEST INFRASTRUCTURE ONLY).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The CUDA library never calls it, and the
two share no code: the C source here (``pkv_oracle.c``) is compiled with gcc
into ``liboracle.so`` and loaded with ctypes.

The arithmetic and the passages it follows are documented at the top of
``pkv_oracle.c``.  This module only marshals torch CPU tensors into the C
calls.  Every function here is pinned against something other than itself
(closed forms, invariants, brute force on tiny inputs, a library routine on
special cases): ``paged_attn`` and ``kv_append`` in
``tests/test_oracle_pins.py``, the packed forms in
``tests/test_oracle_varlen_pins.py``, ``split_partials`` in
``tests/test_oracle_split_pins.py`` and ``paged_attn_bwd`` in
``tests/test_oracle_bwd_pins.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "pkv_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile pkv_oracle.c into liboracle.so with gcc (fp64, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
               "-o", _LIB, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        p = ctypes.c_void_p
        i64 = ctypes.c_int64
        i32 = ctypes.c_int
        lib.oracle_paged_attn.argtypes = [p, p, p, p, p, p, i64, p, i64, i32, p,
                                          i32, i32, i32, i32, i32, i32,
                                          ctypes.c_double, i32,
                                          i32, i32, i32, i32, p, p]
        lib.oracle_paged_attn.restype = i32
        lib.oracle_kv_append.argtypes = [p, p, p, p, p, p, p, p, i64, p, i64,
                                         i32, p, i32, i32, i32, i32, i32]
        lib.oracle_kv_append.restype = i32
        lib.oracle_set_num_threads.argtypes = [i32]
        lib.oracle_set_num_threads.restype = None
        lib.oracle_num_threads.argtypes = []
        lib.oracle_num_threads.restype = i32
        _lib = lib
    return _lib


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def set_num_threads(n: int) -> None:
    _load().oracle_set_num_threads(int(n))


def _strides3(t: torch.Tensor, dims=(0, 1, 2)) -> ctypes.Array:
    return (ctypes.c_int64 * 3)(*[int(t.stride(d)) for d in dims])


def _bits(t: torch.Tensor) -> torch.Tensor:
    if t.dtype != torch.bfloat16 or t.device.type != "cpu":
        raise TypeError("oracle expects bf16 CPU tensors")
    if t.stride(-1) != 1:
        raise ValueError("oracle expects a unit stride on the last (head_dim) axis")
    return t.view(torch.int16)


def paged_attn(q, k_cache, v_cache, block_table, seqlens, scale, causal,
               b_range=None, kvh_range=None):
    """fp64 paged attention.

    q:            [B, sq, Hq, D] bf16 (CPU)
    k_cache/v_cache: [num_blocks, block_size, Hkv, D] bf16 views (any strides,
                  unit stride on D), e.g. the interleaved views kv[:, 0], kv[:, 1]
    block_table:  [B, nblk] int32
    seqlens:      [B] int32, context length including the query tokens
    Returns (out [B, sq, Hq, D] fp64, lse [B, Hq, sq] fp64).  Rows outside
    b_range x kvh_range are left as NaN.  Raises RuntimeError (status 2) when
    a selected sequence has a token past the table's nblk columns or a block
    id outside [0, num_blocks).
    """
    lib = _load()
    B, sq, Hq, D = q.shape
    nblocks, bs, Hkv, D2 = k_cache.shape
    assert D2 == D and tuple(v_cache.shape) == tuple(k_cache.shape)
    qb, kb, vb = _bits(q), _bits(k_cache), _bits(v_cache)
    bt = block_table.to(torch.int32)
    if bt.stride(1) != 1:
        bt = bt.contiguous()
    sl = seqlens.to(torch.int32).contiguous()
    out = torch.full((B, sq, Hq, D), float("nan"), dtype=torch.float64)
    lse = torch.full((B, Hq, sq), float("nan"), dtype=torch.float64)
    b0, b1 = b_range if b_range is not None else (0, B)
    h0, h1 = kvh_range if kvh_range is not None else (0, Hkv)
    rc = lib.oracle_paged_attn(
        qb.data_ptr(), _strides3(q), kb.data_ptr(), _strides3(k_cache),
        vb.data_ptr(), _strides3(v_cache), nblocks, bt.data_ptr(), bt.stride(0), bt.shape[1],
        sl.data_ptr(), B, sq, Hq, Hkv, D, bs, float(scale), int(bool(causal)),
        b0, b1, h0, h1, out.data_ptr(), lse.data_ptr())
    if rc != 0:
        raise RuntimeError(f"oracle_paged_attn failed with status {rc}")
    return out, lse


def kv_append(k_new, v_new, k_cache, v_cache, block_table, seqlens):
    """Write k_new/v_new [B, n, Hkv, D] into the caches (in place) at
    positions seqlens[b] + t, copying bf16 bits unchanged."""
    lib = _load()
    B, n, Hkv, D = k_new.shape
    nblocks, bs, Hkv2, D2 = k_cache.shape
    assert (Hkv2, D2) == (Hkv, D)
    bt = block_table.to(torch.int32)
    if bt.stride(1) != 1:
        bt = bt.contiguous()
    sl = seqlens.to(torch.int32).contiguous()
    rc = lib.oracle_kv_append(
        _bits(k_new).data_ptr(), _strides3(k_new), _bits(v_new).data_ptr(),
        _strides3(v_new), _bits(k_cache).data_ptr(), _strides3(k_cache),
        _bits(v_cache).data_ptr(), _strides3(v_cache), nblocks, bt.data_ptr(),
        bt.stride(0), bt.shape[1], sl.data_ptr(), B, n, Hkv, D, bs)
    if rc != 0:
        raise RuntimeError(f"oracle_kv_append failed with status {rc}")


def paged_attn_varlen(q, k_cache, v_cache, block_table, seqlens, cu_seqlens_q, scale, causal):
    """fp64 attention of packed multi-request queries (the cumulative query
    lengths of a packed forward, AstrAI commit search page: "Pack prompts ...
    into one forward", "Select per-request final logits from cumulative query
    lengths").  Packing is only an indexing convention: request b is the dense
    problem of its own n_b = cu[b+1] - cu[b] queries (the last n_b positions of
    its context), so each request is handed to paged_attn on its own.

    q: [total_q, Hq, D] bf16; cu_seqlens_q: [B + 1] int.  Returns (out
    [total_q, Hq, D] fp64, lse [Hq, total_q] fp64, final_out [B, Hq, D] fp64,
    final_lse [B, Hq] fp64); the final row of request b is its packed token
    cu[b+1] - 1 (NaN for a request with no query)."""
    total_q, Hq, D = q.shape
    cu = [int(x) for x in cu_seqlens_q.tolist()]
    B = len(cu) - 1
    out = torch.full((total_q, Hq, D), float("nan"), dtype=torch.float64)
    lse = torch.full((Hq, total_q), float("nan"), dtype=torch.float64)
    fin_out = torch.full((B, Hq, D), float("nan"), dtype=torch.float64)
    fin_lse = torch.full((B, Hq), float("nan"), dtype=torch.float64)
    for b in range(B):
        a, e = cu[b], cu[b + 1]
        if e <= a:
            continue
        o_b, l_b = paged_attn(q[a:e].unsqueeze(0), k_cache, v_cache, block_table[b:b + 1],
                              seqlens[b:b + 1], scale, causal)
        out[a:e] = o_b[0]
        lse[:, a:e] = l_b[0]
        fin_out[b] = o_b[0, -1]
        fin_lse[b] = l_b[0, :, -1]
    return out, lse, fin_out, fin_lse


def kv_append_varlen(k_new, v_new, k_cache, v_cache, block_table, seqlens, cu_seqlens_new):
    """kv_append for packed new tokens [total_new, Hkv, D]: sequence b's are
    rows cu[b] .. cu[b+1] - 1, written at positions seqlens[b] + t."""
    cu = [int(x) for x in cu_seqlens_new.tolist()]
    for b in range(len(cu) - 1):
        a, e = cu[b], cu[b + 1]
        if e <= a:
            continue
        kv_append(k_new[a:e].unsqueeze(0), v_new[a:e].unsqueeze(0), k_cache, v_cache,
                  block_table[b:b + 1], seqlens[b:b + 1])


def split_partials(q, k_cache, v_cache, block_table, seqlens, scale, causal, split_begin,
                   n_splits_local, split_tokens=4096):
    """fp64 unnormalised partials of the splits [split_begin, split_begin +
    n_splits_local): for every (b, i, h, local split), over the row's visible
    keys j in [split_tokens * s, split_tokens * (s + 1)): m = max_j s_j (natural
    units, s_j = scale * q.k_j), l = sum_j exp(s_j - m), acc = sum_j exp(s_j -
    m) v_j; m = -inf, l = 0, acc = 0 where the row sees no key of the split.
    The KV chunks of the CP forward (RL-Kernel PR #284, Changes: KV chunk
    size, fixed global_block_index merge order).  Plain torch fp64 on the CPU.

    Returns (m [B, sq, Hq, n], l [B, sq, Hq, n], acc [B, sq, Hq, n, D])."""
    B, sq, Hq, D = q.shape
    nb, bs, Hkv, _ = k_cache.shape
    G = Hq // Hkv
    m = torch.full((B, sq, Hq, n_splits_local), float("-inf"), dtype=torch.float64)
    l = torch.zeros((B, sq, Hq, n_splits_local), dtype=torch.float64)
    acc = torch.zeros((B, sq, Hq, n_splits_local, D), dtype=torch.float64)
    for b in range(B):
        n = max(int(seqlens[b]), 0)
        if n == 0:
            continue
        j = torch.arange(n)
        blk = block_table[b, j // bs].long()
        K = k_cache[blk, j % bs].double()    # [n, Hkv, D]
        V = v_cache[blk, j % bs].double()
        for i in range(sq):
            lim = min(n, n - sq + i + 1) if causal else n
            for h in range(Hq):
                if lim <= 0:
                    continue
                s_all = scale * (K[:lim, h // G] @ q[b, i, h].double())
                for ls in range(n_splits_local):
                    a = (split_begin + ls) * split_tokens
                    e = min(a + split_tokens, lim)
                    if e <= a:
                        continue
                    sc = s_all[a:e]
                    mm = float(sc.max())
                    w = torch.exp(sc - mm)
                    m[b, i, h, ls] = mm
                    l[b, i, h, ls] = w.sum()
                    acc[b, i, h, ls] = w @ V[a:e, h // G]
    return m, l, acc


def paged_attn_bwd(q, k_cache, v_cache, block_table, seqlens, scale, causal, dout):
    """fp64 gradients of paged softmax attention (the backward of paged_attn's
    forward, same masks and bottom-right causal alignment), for the
    deterministic prefill backward over the same forward graph (RL-Kernel PR
    #284 "feat(attention): add CP backward drift validation", Changes:
    backward_reference over the same forward, dq / dk / dv).  With
    p_ij = exp(s_ij - lse_i), s_ij = scale * q_i.k_j over the visible keys:
        D_i  = sum_j p_ij (dout_i . v_j)      (= dout_i . out_i)
        ds_ij = p_ij (dout_i . v_j - D_i)
        dq_i = scale * sum_j ds_ij k_j
        dk_j = scale * sum_i ds_ij q_i,   dv_j = sum_i p_ij dout_i
    summed over every query row (token and query head of the KV head's group)
    that sees key j.  Plain torch fp64 on the CPU.

    Returns (dq [B, sq, Hq, D], dk [B, Lmax, Hkv, D], dv [B, Lmax, Hkv, D])
    with dk / dv indexed by token position (zeros past seqlens[b])."""
    B, sq, Hq, D = q.shape
    nb, bs, Hkv, _ = k_cache.shape
    G = Hq // Hkv
    Lmax = max(int(x) for x in seqlens) if len(seqlens) else 0
    dq = torch.zeros(B, sq, Hq, D, dtype=torch.float64)
    dk = torch.zeros(B, max(Lmax, 1), Hkv, D, dtype=torch.float64)
    dv = torch.zeros(B, max(Lmax, 1), Hkv, D, dtype=torch.float64)
    for b in range(B):
        n = max(int(seqlens[b]), 0)
        if n == 0:
            continue
        j = torch.arange(n)
        blk = block_table[b, j // bs].long()
        K = k_cache[blk, j % bs].double()    # [n, Hkv, D]
        V = v_cache[blk, j % bs].double()
        for h in range(Hq):
            g = h // G
            Q = q[b, :, h].double()          # [sq, D]
            dO = dout[b, :, h].double()
            S = scale * (Q @ K[:, g].T)      # [sq, n]
            pos = n - sq + torch.arange(sq)
            vis = torch.arange(n)[None, :] < n
            if causal:
                vis = vis & (torch.arange(n)[None, :] <= pos[:, None])
            S = S.masked_fill(~vis, float("-inf"))
            m = S.max(dim=1, keepdim=True).values
            has = torch.isfinite(m)
            m = torch.where(has, m, torch.zeros_like(m))
            E = torch.exp(S - m) * vis
            P = E / E.sum(dim=1, keepdim=True).clamp_min(1e-300)
            P = P * has
            dP = dO @ V[:, g].T              # [sq, n]
            Dv = (P * dP).sum(dim=1, keepdim=True)
            dS = P * (dP - Dv)
            dq[b, :, h] = scale * (dS @ K[:, g])
            dk[b, :n, g] += scale * (dS.T @ Q)
            dv[b, :n, g] += P.T @ dO
    return dq, dk, dv
