"""Ring attention across real ranks: one process per GPU, K/V blocks passed around
the ring with torch.distributed point-to-point transfers.

"上下文并行与 Ring Attention" (hs-black.github.io), section Ring Attention: N
devices form a ring; device i starts with Q_i, K_i, V_i; at step r it attends its
Q to the K/V block it holds (the block of rank (i - r) mod N), merges the partial
into its running (o, lse), and passes the block on to device i + 1 while it
receives the next one from device i - 1, so the transfer hides behind the
computation.  Q and O never move.

Each rank holds its c = S / N tokens in the layout's order (rank-major local
blocks, as cp_layout_permute produces them on one device).  The step's compute is
cp_block_attn_fwd with the rank ranges of the layout: the first step writes the
fp32 (o, lse), later steps merge into them with the kernel's fused epilogue.  The
exchange of the next block is posted before the compute and waited for after it.

The backward (ring_attn_bwd_dist) walks the same ring once more (section 分块注意力,
paragraph on the backward pass): at step r rank i holds block (i - r) mod N together
with that block's travelling fp32 dK, dV accumulators, adds its queries' shares to
its own dQ and to the travelling dK, dV (cp_block_attn_bwd, with the rows' global
lse and o from the forward), and passes block and accumulators on.  The next K/V
block is posted before the compute; the accumulators can only leave after it.
After the last step every accumulator is one hop from its owner, and one more
exchange brings it home.

ring_attn_fwd_peer runs the same forward schedule with no rank sending: the ranks
of one node map each other's K/V blocks into their own address space once
(PeerBlocks, CUDA IPC through the library's cp_peer_* calls), and step r pulls rank
(i - r) mod N's block into a local buffer one step ahead with the copy engines,
overlapped with the step before (or, with stage=False, the block kernel reads it
where it lies).  No collective sits on the data path.  At each step the N ranks
pull N different blocks (a permutation), so every link carries one block.  ring_attn_bwd_peer does the same for the
backward: step r adds rank i's shares for block (i - r) mod N into that block
owner's fp32 dK, dV accumulators where they lie, with a host barrier between steps
so that each accumulator has one writer at a time.

The compute steps can be replaced (`compute=`), which is how the schedules are
tested on CPU ranks (gloo) without a GPU.
"""
import torch
import torch.distributed as dist

from . import _binding as B


def _nvtx_push(t, name):
    """An NVTX range per ring step for profilers (CUDA tensors only)."""
    if t.is_cuda:
        torch.cuda.nvtx.range_push(name)


def _nvtx_pop(t):
    if t.is_cuda:
        torch.cuda.nvtx.range_pop()


def block_compute(q, k, v, q_range, kv_range, causal, scale, o, lse, accumulate):
    """The default step: the tensor-core (bf16) or FFMA (fp32) block kernel."""
    B.block_attn_fwd(q, k, v, q_range, kv_range, causal, scale, o, lse, accumulate=accumulate)


def merge_out(o_acc, lse_acc, o_b, lse_b, o_out):
    """The default last merge: the standalone LSE-merge kernel writing o in the
    output dtype."""
    B.lse_merge(o_acc, lse_acc, o_b, lse_b, o_out=o_out)


def ring_attn_fwd_dist(q, k, v, layout, causal, scale=None, group=None, compute=block_compute, merge=merge_out):
    """This rank's share of ring attention.

    q [b, c, Hq, d], k / v [b, c, Hkv, d]: this rank's local blocks (its layout
    positions, in order).  Returns (o [b, c, Hq, d] in q's dtype, lse [b, Hq, c]
    fp32) for the local queries.  All ranks of `group` call it together.

    Steps 0 .. N-2 keep the running (o, lse) in fp32 (the block kernel's fused
    merge from step 1 on); the last step writes its partial and the standalone
    merge folds it in and writes o in q's dtype.
    """
    rank = dist.get_rank(group)
    N = dist.get_world_size(group)
    b, c, Hq, d = q.shape
    if scale is None:
        scale = 0.0  # the library's default: 1/sqrt(d)
    S = c * N
    q_range = B.layout_range(layout, N, S, rank)
    nxt, prv = (rank + 1) % N, (rank - 1) % N
    to_global = (lambda r: dist.get_global_rank(group, r)) if group is not None else (lambda r: r)
    out = torch.empty((b, c, Hq, d), dtype=q.dtype, device=q.device)
    lse = torch.empty((b, Hq, c), dtype=torch.float32, device=q.device)
    if N == 1:
        compute(q, k, v, q_range, q_range, causal, scale, out, lse, False)
        return out, lse
    o = torch.empty((b, c, Hq, d), dtype=torch.float32, device=q.device)
    # the caller's k, v are only read (step 0); received blocks alternate between two
    # buffers of the driver's own
    cur_k, cur_v = k.contiguous(), v.contiguous()
    bufs = [(torch.empty_like(cur_k), torch.empty_like(cur_v)) for _ in range(min(2, N - 1))]
    for r in range(N):
        _nvtx_push(q, "ring step %d of %d" % (r, N))
        src = (rank - r) % N                      # the block this rank holds at step r
        reqs = []
        if r + 1 < N:                             # pass the block on, take the next one
            buf_k, buf_v = bufs[r % 2]
            ops = [dist.P2POp(dist.isend, cur_k, to_global(nxt), group),
                   dist.P2POp(dist.isend, cur_v, to_global(nxt), group),
                   dist.P2POp(dist.irecv, buf_k, to_global(prv), group),
                   dist.P2POp(dist.irecv, buf_v, to_global(prv), group)]
            reqs = dist.batch_isend_irecv(ops)
        kv_range = B.layout_range(layout, N, S, src)
        if r + 1 < N:
            compute(q, cur_k, cur_v, q_range, kv_range, causal, scale, o, lse, r > 0)
        else:
            o_b = torch.empty_like(out)
            lse_b = torch.empty_like(lse)
            compute(q, cur_k, cur_v, q_range, kv_range, causal, scale, o_b, lse_b, False)
            merge(o, lse, o_b, lse_b, out)
        for req in reqs:
            req.wait()
        if r + 1 < N:
            cur_k, cur_v = buf_k, buf_v
        _nvtx_pop(q)
    return out, lse


def block_bwd_compute(q, k, v, o, lse, do, q_range, kv_range, causal, scale, dq_acc, dk_acc, dv_acc):
    """The default backward step: the block backward, adding into fp32 accumulators."""
    B.block_attn_bwd(q, k, v, o, lse, do, q_range, kv_range, causal, scale, dq_acc, dk_acc, dv_acc)


def ring_attn_bwd_dist(q, k, v, o, lse, do, layout, causal, scale=None, group=None, compute=block_bwd_compute):
    """This rank's gradients of ring attention.

    q, o, do [b, c, Hq, d], k / v [b, c, Hkv, d]: this rank's local blocks; o and lse
    [b, Hq, c] are this rank's results of the whole-sequence forward (for example
    ring_attn_fwd_dist).  Returns (dq, dk, dv) in q's dtype for the local blocks.
    All ranks of `group` call it together.
    """
    import torch
    rank = dist.get_rank(group)
    N = dist.get_world_size(group)
    b, c, Hq, d = q.shape
    if scale is None:
        scale = 0.0  # the library's default: 1/sqrt(d)
    S = c * N
    q_range = B.layout_range(layout, N, S, rank)
    nxt, prv = (rank + 1) % N, (rank - 1) % N
    to_global = (lambda r: dist.get_global_rank(group, r)) if group is not None else (lambda r: r)

    def exchange(send, recv):
        ops = [dist.P2POp(dist.isend, t, to_global(nxt), group) for t in send]
        ops += [dist.P2POp(dist.irecv, t, to_global(prv), group) for t in recv]
        return dist.batch_isend_irecv(ops)

    dq = torch.zeros(q.shape, dtype=torch.float32, device=q.device)
    # the caller's k, v are only read (step 0); received blocks alternate between two
    # buffers of the driver's own
    cur_k, cur_v = k.contiguous(), v.contiguous()
    bufs = [(torch.empty_like(cur_k), torch.empty_like(cur_v)) for _ in range(min(2, N - 1))]
    # the travelling accumulators live where the travelling block does
    f32 = dict(dtype=torch.float32, device=k.device)
    cur_dk, cur_dv = torch.zeros(k.shape, **f32), torch.zeros(v.shape, **f32)
    buf_dk, buf_dv = torch.empty_like(cur_dk), torch.empty_like(cur_dv)
    for r in range(N):
        _nvtx_push(q, "ring backward step %d of %d" % (r, N))
        src = (rank - r) % N                      # the block this rank holds at step r
        if r + 1 < N:
            buf_k, buf_v = bufs[r % 2]
        kv_reqs = exchange([cur_k, cur_v], [buf_k, buf_v]) if r + 1 < N else []
        compute(q, cur_k, cur_v, o, lse, do, q_range, B.layout_range(layout, N, S, src), causal, scale, dq,
                cur_dk, cur_dv)
        # the block's accumulators follow it; after the last step they go home
        acc_reqs = exchange([cur_dk, cur_dv], [buf_dk, buf_dv]) if N > 1 else []
        for req in kv_reqs + acc_reqs:
            req.wait()
        if N > 1:
            cur_dk, buf_dk = buf_dk, cur_dk
            cur_dv, buf_dv = buf_dv, cur_dv
            if r + 1 < N:
                cur_k, cur_v = buf_k, buf_v
        _nvtx_pop(q)
    return dq.to(q.dtype), cur_dk.to(k.dtype), cur_dv.to(v.dtype)


class PeerBlocks:
    """Per-rank blocks that the kernels of every rank of `group` read and write in place.

    shapes, dtype, device: this rank's blocks (for the ring: K and V, [b, c, Hkv, d]
    each; or the fp32 dK, dV accumulators).  `local[t]` is this rank's block t, for
    the caller to write (copy_, or as the output of the step producing it);
    `views[t][j]` is rank j's block t as a tensor of this process -- rank j's memory,
    mapped, not a copy (this rank's own tensor for j == rank).  Every rank of the
    group constructs it together.

    Order of use, every rank alike: write `local`, publish() (the writes are finished
    everywhere), run the kernels that use `views`, release() (that work is finished
    everywhere) before a block is written again; close() at the end.  The ring
    functions below call publish() and release() themselves.

    CUDA blocks come from torch's caching allocator (cudaMalloc'd memory) and are
    mapped with cp_peer_export / cp_peer_import, once, here.  CPU blocks (the gloo
    tests) live in POSIX shared memory opened by every rank, so a peer's view is the
    same memory there too."""

    def __init__(self, shapes, dtype, device, group=None):
        self.group = group
        self.rank, self.N = dist.get_rank(group), dist.get_world_size(group)
        self.device = torch.device(device)
        self._handles, self._shm = [], []
        shapes = [tuple(sh) for sh in shapes]
        if self.device.type == "cuda":
            self.local = [torch.empty(sh, dtype=dtype, device=self.device) for sh in shapes]
            mine = [B.peer_export(t) for t in self.local]
        else:
            self.local, mine = [], []
            for sh in shapes:
                t, name = self._shared_cpu(sh, dtype, None)
                self.local.append(t)
                mine.append(name)
        everyone = [None] * self.N
        dist.all_gather_object(everyone, mine, group=group)
        self.views = [[None] * self.N for _ in shapes]
        for j, handles in enumerate(everyone):
            for t, (h, sh) in enumerate(zip(handles, shapes)):
                if j == self.rank:
                    self.views[t][j] = self.local[t]
                elif self.device.type == "cuda":
                    self.views[t][j] = B.peer_import(h, sh, dtype)
                    self._handles.append(h)
                else:
                    self.views[t][j] = self._shared_cpu(sh, dtype, h)[0]

    def _shared_cpu(self, shape, dtype, name):
        """A CPU tensor in POSIX shared memory: a new segment (name None) or the
        segment another rank made."""
        from multiprocessing import resource_tracker, shared_memory
        nbytes = max(1, torch.Size(shape).numel() * torch.empty((), dtype=dtype).element_size())
        if name is None:
            shm = shared_memory.SharedMemory(create=True, size=nbytes)
        else:
            shm = shared_memory.SharedMemory(name=name)
            resource_tracker.unregister(shm._name, "shared_memory")  # the creating rank unlinks it
        self._shm.append((shm, name is None))
        return torch.frombuffer(shm.buf, dtype=dtype, count=torch.Size(shape).numel()).view(shape), shm.name

    def _sync(self):
        if self.device.type == "cuda":
            torch.cuda.current_stream(self.device).synchronize()
        dist.barrier(group=self.group)

    def publish(self):
        """Every rank's blocks are written: this rank's queued work finishes, then the
        ranks meet on the host."""
        self._sync()

    def release(self):
        """Every rank's work on the blocks is finished: this rank's queued work
        finishes, then the ranks meet on the host."""
        self._sync()

    def close(self):
        """release(), then every rank drops its mappings of the others' blocks before
        any block is freed.  Tensors taken from `views` or `local` must not be used
        after close(): the memory behind them is unmapped or freed."""
        self.release()
        for h in self._handles:
            B.peer_close(h)
        self._handles = []
        self.views = None
        self.local = None
        dist.barrier(group=self.group)
        for shm, owner in self._shm:
            try:
                shm.close()
            except BufferError:  # a caller still holds a view; the mapping goes at exit
                pass
            if owner:
                shm.unlink()
        self._shm = []


def ring_attn_fwd_peer(q, kv, layout, causal, scale=None, stage=True, compute=block_compute, merge=merge_out):
    """This rank's share of ring attention over blocks that no rank sends.

    q [b, c, Hq, d]: this rank's local queries (its layout positions, in order);
    kv: a PeerBlocks over the group whose local blocks 0 and 1 hold this rank's K and
    V [b, c, Hkv, d], already written.  Returns (o [b, c, Hq, d] in q's dtype, lse
    [b, Hq, c] fp32) for the local queries.  All ranks of the group call it
    together.

    Step r attends to rank (i - r) mod N's block.  stage=True pulls that block into
    one of two local buffers one step ahead, on a copy stream with the copy engines
    (cp_peer_copy), while the block kernel of the step before runs: every CTA of the
    forward reads every K/V tile of the block, so reading the peer in place would
    carry each tile across the link once per reading CTA.  stage=False runs the block
    kernel on the peer's memory directly (the same GPU's memory when the ranks share
    one, as in the tests).  Steps 0 .. N-2 keep the running (o, lse) in fp32 (the
    block kernel's fused merge from step 1 on), and the last step's partial is
    folded in by the standalone merge, which writes o in q's dtype.
    """
    rank, N = kv.rank, kv.N
    ks, vs = kv.views[0], kv.views[1]
    b, c, Hq, d = q.shape
    if scale is None:
        scale = 0.0  # the library's default: 1/sqrt(d)
    S = c * N
    q_range = B.layout_range(layout, N, S, rank)
    out = torch.empty((b, c, Hq, d), dtype=q.dtype, device=q.device)
    lse = torch.empty((b, Hq, c), dtype=torch.float32, device=q.device)
    kv.publish()
    if N == 1:
        compute(q, ks[0], vs[0], q_range, q_range, causal, scale, out, lse, False)
        kv.release()
        return out, lse
    cuda = q.is_cuda
    if stage:
        # steps 1 .. N-1 read block (rank - r) mod N from buffer (r - 1) % n_buf
        n_buf = min(2, N - 1)
        bufs = [(torch.empty_like(ks[rank]), torch.empty_like(vs[rank])) for _ in range(n_buf)]
        if cuda:
            main, side = torch.cuda.current_stream(), torch.cuda.Stream()
            fetched = [torch.cuda.Event() for _ in range(n_buf)]
            used = [torch.cuda.Event() for _ in range(n_buf)]

    def fetch(r):
        """Pull block (rank - r) mod N into its buffer, after the step that last read
        that buffer (step r - n_buf) is done with it."""
        src, slot = (rank - r) % N, (r - 1) % n_buf
        if not cuda:
            bufs[slot][0].copy_(ks[src])
            bufs[slot][1].copy_(vs[src])
            return
        with torch.cuda.stream(side):
            if r - n_buf >= 1:
                side.wait_event(used[slot])
            B.peer_copy(bufs[slot][0], ks[src])
            B.peer_copy(bufs[slot][1], vs[src])
            fetched[slot].record(side)

    o = torch.empty((b, c, Hq, d), dtype=torch.float32, device=q.device)
    if stage:
        fetch(1)
    for r in range(N):
        _nvtx_push(q, "peer ring step %d of %d" % (r, N))
        src = (rank - r) % N                      # the block step r attends to
        kv_range = B.layout_range(layout, N, S, src)
        if r == 0 or not stage:
            kk, vv = ks[src], vs[src]             # the local block, or the peer's where it lies
        else:
            slot = (r - 1) % n_buf
            if cuda:
                main.wait_event(fetched[slot])
            kk, vv = bufs[slot]
            if r + 1 < N:
                fetch(r + 1)                      # the next block comes in while this step runs
        if r + 1 < N:
            compute(q, kk, vv, q_range, kv_range, causal, scale, o, lse, r > 0)
        else:
            o_b = torch.empty_like(out)
            lse_b = torch.empty_like(lse)
            compute(q, kk, vv, q_range, kv_range, causal, scale, o_b, lse_b, False)
            merge(o, lse, o_b, lse_b, out)
        if stage and cuda and r >= 1:
            used[(r - 1) % n_buf].record(main)
        _nvtx_pop(q)
    if stage and cuda:
        main.wait_stream(side)
    kv.release()
    return out, lse


def ring_attn_bwd_peer(q, kv, o, lse, do, layout, causal, scale=None, acc=None, compute=block_bwd_compute):
    """This rank's gradients of ring attention with every block left in place.

    q, o, do [b, c, Hq, d]: this rank's local blocks; o and lse [b, Hq, c] are this
    rank's results of the whole-sequence forward (for example ring_attn_fwd_peer);
    kv: the PeerBlocks holding every rank's K and V (blocks 0 and 1), already
    written; acc: a PeerBlocks of two blocks shaped like K and V in the accumulation
    dtype (fp32 for the kernels) over the same group, reused across calls (made and
    closed here when None).  Returns (dq, dk, dv) in q's / k's dtype for this
    rank's blocks.  All ranks of the group call it together.

    Step r: rank i adds its queries' shares for block j = (i - r) mod N into its own
    dQ and into rank j's dK, dV accumulators, in rank j's memory (the block backward
    adds with plain fp32 loads and stores).  The ranks meet on the host after every
    step, so at every step each accumulator has exactly one writer, and the
    accumulators never travel."""
    rank, N = kv.rank, kv.N
    ks, vs = kv.views[0], kv.views[1]
    b, c, Hq, d = q.shape
    if scale is None:
        scale = 0.0  # the library's default: 1/sqrt(d)
    S = c * N
    q_range = B.layout_range(layout, N, S, rank)
    own_acc = acc is None
    if own_acc:
        acc = PeerBlocks([ks[rank].shape, vs[rank].shape], torch.float32, q.device, kv.group)
    acc.local[0].zero_()
    acc.local[1].zero_()
    dq = torch.zeros(q.shape, dtype=acc.local[0].dtype, device=q.device)
    kv.publish()                                  # K, V written and the accumulators zeroed everywhere
    for r in range(N):
        _nvtx_push(q, "peer ring backward step %d of %d" % (r, N))
        src = (rank - r) % N                      # the block step r works on, where it lies
        compute(q, ks[src], vs[src], o, lse, do, q_range, B.layout_range(layout, N, S, src), causal, scale, dq,
                acc.views[0][src], acc.views[1][src])
        acc.release()                             # this step's adds are finished everywhere
        _nvtx_pop(q)
    dk = acc.local[0].to(ks[rank].dtype, copy=True)  # a copy: the accumulators stay with `acc`
    dv = acc.local[1].to(vs[rank].dtype, copy=True)
    if own_acc:
        acc.close()
    return dq.to(q.dtype), dk, dv
