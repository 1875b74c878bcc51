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
"""
from collections import deque


class RefAllocError(Exception):
    def __init__(self, kind: str, msg: str = ""):
        super().__init__(f"{kind}: {msg}")
        self.kind = kind  # 'inval' | 'nomem'


class RefAllocator:
    def __init__(self, num_blocks: int, free_order=None, block_size: int = 16):
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

    # -- sequences ---------------------------------------------------------
    def add_seq(self, sid: int) -> None:
        if sid in self.tables:
            raise RefAllocError("inval", f"sequence {sid} exists")
        self.tables[sid] = []
        self.lengths[sid] = 0

    def fork(self, parent: int, child: int) -> None:
        if parent not in self.tables or child in self.tables:
            raise RefAllocError("inval", f"fork {parent}->{child}")
        self.tables[child] = list(self.tables[parent])
        self.lengths[child] = self.lengths[parent]
        for blk in self.tables[child]:
            self.refcount[blk] += 1

    def free_seq(self, sid: int) -> None:
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
