"""Reference host block allocator (oracle only), in plain Python.

What the pages fix:
* blocks are handed out on demand as a sequence grows, never preallocated,
  and return to the pool when the request ends ("vLLM + PagedAttention：
  打造高并发LLM推理引擎", "它是怎么工作的", items 1, 2 and 4);
* each request keeps a page table from logical page to physical block; the
  blocks need not be contiguous ("PagedAttention 与 vLLM 推理加速" §2.3);
* requests with a common prefix map the same physical blocks; a shared block
  is copied only when a writer appends to it (ibid. §3.2(3); "LLM Systems 24
  ..." §3: reference counts and copy-on-write).

What the pages leave open, read the plainest deterministic way:
* the free list is FIFO: it starts in ``free_order`` (0..n-1 when not
  given), allocation pops the front, a block whose count drops to zero is
  pushed to the back;
* ``free_seq`` releases a table's blocks in table order;
* ``fork`` gives the child a copy of the parent's table and length and adds
  one reference to every block in it;
* appending at position p (0-based): if p is a multiple of the block size
  (no last block, or the last block is full) a fresh block is appended to
  the table; otherwise, if the last block is shared (count > 1), a fresh
  block replaces it in the table, one reference is dropped from the old
  one, and the pair (old, new) is returned for the caller to copy;
  otherwise the token goes into the last block as is.  A full shared block
  is never copied;
* slot = physical block * block_size + offset;
* a call that fails (unknown or duplicate id, pool exhausted) raises and
  leaves every piece of state as it was.

Preemption by swapping ("LLM Systems 24 ..." §3, conclusion: when the pool
runs out of KV blocks a request is preempted and later swapped back in or
recomputed).  The pages give no policy; the readings taken here:
* a second, host-side pool of ``num_host_blocks`` blocks with its own FIFO
  free list (0..n-1) and reference counts;
* ``swap_out(ids)`` moves the listed resident sequences to the host pool:
  every distinct device block their tables hold (in id order, then table
  order) gets one host block, and the pair (device, host) is returned for
  the caller to copy; a block that several listed sequences share maps to
  one host block that they share; each holder drops one device reference
  and a device block whose count reaches zero goes to the back of the
  device free list (blocks shared with sequences not listed stay where
  they are, still held by those);
* ``swap_in(ids)`` is the mirror image: every distinct host block of the
  listed swapped sequences gets a fresh device block (pair (host, device)),
  host references are dropped the same way;
* both are all or nothing; a swapped sequence can only be freed or swapped
  in (no append, fork or step);
* the copies of a swap-out must run before anything writes the device
  blocks it released; those of a swap-in before the sequence is read.
"""
from collections import deque


class RefAllocError(Exception):
    def __init__(self, kind: str, msg: str = ""):
        super().__init__(f"{kind}: {msg}")
        self.kind = kind  # 'inval' | 'nomem'


class RefAllocator:
    def __init__(self, num_blocks: int, free_order=None, block_size: int = 16, num_host_blocks: int = 0):
        if free_order is None:
            free_order = range(num_blocks)
        free_order = [int(x) for x in free_order]
        if sorted(free_order) != list(range(num_blocks)):
            raise RefAllocError("inval", "free_order must be a permutation of 0..num_blocks-1")
        self.num_blocks = num_blocks
        self.block_size = block_size
        self.free = deque(free_order)
        self.refcount = [0] * num_blocks
        self.tables = {}  # seq id -> list of physical blocks
        self.lengths = {}  # seq id -> number of tokens
        self.num_host_blocks = num_host_blocks
        self.host_free = deque(range(num_host_blocks))
        self.host_refcount = [0] * num_host_blocks
        self.swapped = {}  # seq id -> (list of host blocks, number of tokens)

    # -- sequences ---------------------------------------------------------
    def add_seq(self, sid: int) -> None:
        if sid in self.tables or sid in self.swapped:
            raise RefAllocError("inval", f"sequence {sid} exists")
        self.tables[sid] = []
        self.lengths[sid] = 0

    def fork(self, parent: int, child: int) -> None:
        if parent not in self.tables or child in self.tables or child in self.swapped:
            raise RefAllocError("inval", f"fork {parent}->{child}")
        self.tables[child] = list(self.tables[parent])
        self.lengths[child] = self.lengths[parent]
        for blk in self.tables[child]:
            self.refcount[blk] += 1

    def free_seq(self, sid: int) -> None:
        if sid in self.swapped:
            for blk in self.swapped.pop(sid)[0]:
                self.host_refcount[blk] -= 1
                if self.host_refcount[blk] == 0:
                    self.host_free.append(blk)
            return
        if sid not in self.tables:
            raise RefAllocError("inval", f"unknown sequence {sid}")
        for blk in self.tables.pop(sid):
            self.refcount[blk] -= 1
            if self.refcount[blk] == 0:
                self.free.append(blk)
        del self.lengths[sid]

    # -- appends -----------------------------------------------------------
    def _needs_block(self, sid: int, refcount_of) -> bool:
        pos = self.lengths[sid]
        if pos % self.block_size == 0:
            return True
        return refcount_of(self.tables[sid][-1]) > 1

    def append_slot(self, sid: int):
        """Append one token; return (slot, cow) with cow = (src, dst) or None."""
        if sid not in self.tables:
            raise RefAllocError("inval", f"unknown sequence {sid}")
        if self._needs_block(sid, lambda b: self.refcount[b]) and not self.free:
            raise RefAllocError("nomem", "pool exhausted")
        return self._append_unchecked(sid)

    def _append_unchecked(self, sid: int):
        table = self.tables[sid]
        pos = self.lengths[sid]
        page, off = divmod(pos, self.block_size)
        cow = None
        if off == 0:
            blk = self.free.popleft()
            self.refcount[blk] = 1
            table.append(blk)
        elif self.refcount[table[-1]] > 1:
            src = table[-1]
            dst = self.free.popleft()
            self.refcount[dst] = 1
            self.refcount[src] -= 1
            table[-1] = dst
            cow = (src, dst)
        self.lengths[sid] = pos + 1
        return table[page] * self.block_size + off, cow

    def append_tokens(self, sid: int, n: int):
        """Append n tokens one by one; return (slots, cows).  All or nothing."""
        if sid not in self.tables:
            raise RefAllocError("inval", f"unknown sequence {sid}")
        need = 0
        pos = self.lengths[sid]
        shared_last = pos % self.block_size != 0 and self.refcount[self.tables[sid][-1]] > 1
        for i in range(n):
            p = pos + i
            if p % self.block_size == 0 or (i == 0 and shared_last):
                need += 1
        if need > len(self.free):
            raise RefAllocError("nomem", "pool exhausted")
        slots, cows = [], []
        for _ in range(n):
            s, c = self._append_unchecked(sid)
            slots.append(s)
            if c is not None:
                cows.append(c)
        return slots, cows

    def step(self, sids):
        """One decode step: append one token to each listed sequence in order.

        Returns (slots, cow_pairs).  Ids must be distinct and known.  All or
        nothing: if the pool cannot serve every append, nothing changes.
        """
        sids = list(sids)
        if len(set(sids)) != len(sids) or any(s not in self.tables for s in sids):
            raise RefAllocError("inval", "step ids must be distinct, known sequences")
        # count the blocks the step takes, tracking the drops CoW makes to
        # the counts of blocks that later entries may share
        drops = {}
        need = 0
        for s in sids:
            if self._needs_block(s, lambda b: self.refcount[b] - drops.get(b, 0)):
                need += 1
                if self.lengths[s] % self.block_size != 0:
                    last = self.tables[s][-1]
                    drops[last] = drops.get(last, 0) + 1
        if need > len(self.free):
            raise RefAllocError("nomem", "pool exhausted")
        slots, cows = [], []
        for s in sids:
            slot, c = self._append_unchecked(s)
            slots.append(slot)
            if c is not None:
                cows.append(c)
        return slots, cows

    # -- preemption by swapping ------------------------------------------------
    @staticmethod
    def _move(sids, table_of, src_ref, src_free, dst_ref, dst_free):
        """Give every distinct block of the listed tables a block popped from
        dst_free; drop the holders' references on the source side.  Returns
        (pairs, new tables).  The caller has checked that dst_free suffices."""
        mapping, pairs, tables = {}, [], []
        for s in sids:
            new = []
            for blk in table_of(s):
                if blk not in mapping:
                    mapping[blk] = dst_free.popleft()
                    pairs.append((blk, mapping[blk]))
                new.append(mapping[blk])
            tables.append(new)
        for s, new in zip(sids, tables):
            for blk, nb in zip(table_of(s), new):
                dst_ref[nb] += 1
                src_ref[blk] -= 1
                if src_ref[blk] == 0:
                    src_free.append(blk)
        return pairs, tables

    def swap_out(self, sids):
        """Move resident sequences to the host pool; return the (device block,
        host block) pairs to copy.  All or nothing."""
        sids = list(sids)
        if len(set(sids)) != len(sids) or any(s not in self.tables for s in sids):
            raise RefAllocError("inval", "swap_out ids must be distinct, resident sequences")
        need = len({b for s in sids for b in self.tables[s]})
        if need > len(self.host_free):
            raise RefAllocError("nomem", "host pool exhausted")
        pairs, tables = self._move(sids, lambda s: self.tables[s], self.refcount, self.free, self.host_refcount,
                                   self.host_free)
        for s, t in zip(sids, tables):
            self.swapped[s] = (t, self.lengths.pop(s))
            del self.tables[s]
        return pairs

    def swap_in(self, sids):
        """Bring swapped sequences back to the device pool; return the (host
        block, device block) pairs to copy.  All or nothing."""
        sids = list(sids)
        if len(set(sids)) != len(sids) or any(s not in self.swapped for s in sids):
            raise RefAllocError("inval", "swap_in ids must be distinct, swapped sequences")
        need = len({b for s in sids for b in self.swapped[s][0]})
        if need > len(self.free):
            raise RefAllocError("nomem", "pool exhausted")
        pairs, tables = self._move(sids, lambda s: self.swapped[s][0], self.host_refcount, self.host_free,
                                   self.refcount, self.free)
        for s, t in zip(sids, tables):
            self.tables[s] = t
            self.lengths[s] = self.swapped.pop(s)[1]
        return pairs

    def host_state(self):
        """(host free list in order, host refcount of every host block)."""
        return list(self.host_free), list(self.host_refcount)

    def swapped_table(self, sid: int):
        t, n = self.swapped[sid]
        return list(t), n

    # -- views ---------------------------------------------------------------
    def block_table(self, sid: int):
        return list(self.tables[sid]), self.lengths[sid]

    def state(self):
        """(free list in order, refcount of every block)."""
        return list(self.free), list(self.refcount)

    def used_slots(self) -> int:
        return sum(self.lengths.values())

    def allocated_slots(self) -> int:
        """Slots of every block some table holds (shared blocks once)."""
        return (self.num_blocks - len(self.free)) * self.block_size
