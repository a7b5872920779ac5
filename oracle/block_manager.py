"""Plain-Python oracle of the KV block manager (test infrastructure only).

Follows the pages step by step:
  * polomodov.tech "vLLM and PagedAttention", slide 12: one shared pool; a
    free block goes to whoever needs it next.  Policy fixed here (the pages
    leave it open): the pool is a stack; a fresh pool hands out 0, 1, 2, ...
    and a freed block is handed out next.
  * slide 11: a new block only when the last block is full; otherwise the new
    token takes the next free slot of the last block.
  * comfyai.app "6.4 PagedAttention", 6.4.2-6.4.3 and slide 13: forked
    sequences share blocks with reference counts; writing into a shared block
    first copies it: the writer gets a new block (count 1), the old block's
    count drops by one; only that last block is copied.
  * slide 15: preemption is all-or-nothing and a preempted request comes
    back by swapping (or recomputation).  A swap moves a group of sequences
    that holds every reference to its blocks to a second (host) pool: each
    distinct block, in order of first appearance (sequences in the given
    order, tables front to back), takes one block of the other pool and
    keeps its reference count; the released blocks go back to their pool's
    stack in that same order.
Slots are physical_block * block_size + offset.
"""
from __future__ import annotations


class OutOfBlocks(Exception):
    pass


class BlockManagerOracle:
    def __init__(self, num_blocks: int, block_size: int, num_cpu_blocks: int = 0):
        self.block_size = block_size
        self.free = list(range(num_blocks - 1, -1, -1))   # pop() gives 0, 1, 2, ...
        self.ref = [0] * num_blocks
        self.cpu_free = list(range(num_cpu_blocks - 1, -1, -1))
        self.cpu_ref = [0] * num_cpu_blocks
        self.tables: dict[int, list[int]] = {}
        self.lens: dict[int, int] = {}
        self.swapped: set[int] = set()

    def _take(self) -> int:
        b = self.free.pop()
        self.ref[b] = 1
        return b

    def num_free(self) -> int:
        return len(self.free)

    def add_sequence(self, seq: int, prompt_len: int):
        if seq in self.tables or prompt_len < 0:
            raise KeyError(seq)
        need = -(-prompt_len // self.block_size)
        if need > len(self.free):
            raise OutOfBlocks
        self.tables[seq] = [self._take() for _ in range(need)]
        self.lens[seq] = prompt_len

    def fork(self, parent: int, child: int):
        if parent not in self.tables or parent in self.swapped or child in self.tables:
            raise KeyError(child)
        self.tables[child] = list(self.tables[parent])
        self.lens[child] = self.lens[parent]
        for b in self.tables[child]:
            self.ref[b] += 1

    def free_sequence(self, seq: int):
        ref, free = (self.cpu_ref, self.cpu_free) if seq in self.swapped else (self.ref, self.free)
        for b in self.tables.pop(seq):
            ref[b] -= 1
            if ref[b] == 0:
                free.append(b)
        del self.lens[seq]
        self.swapped.discard(seq)

    def _move(self, seqs, to_cpu: bool):
        if len(set(seqs)) != len(seqs) or not seqs:
            raise KeyError(seqs)
        for s in seqs:
            if s not in self.tables or (s in self.swapped) == to_cpu:
                raise KeyError(s)
        src_ref, src_free = (self.ref, self.free) if to_cpu else (self.cpu_ref, self.cpu_free)
        dst_ref, dst_free = (self.cpu_ref, self.cpu_free) if to_cpu else (self.ref, self.free)
        order, holders = [], {}
        for s in seqs:
            for b in self.tables[s]:
                if b not in holders:
                    order.append(b)
                holders[b] = holders.get(b, 0) + 1
        if any(src_ref[b] != n for b, n in holders.items()):
            raise KeyError("group shares blocks with other sequences")
        if len(order) > len(dst_free):
            raise OutOfBlocks
        moved, pairs = {}, []
        for b in order:
            nb = dst_free.pop()
            dst_ref[nb] = src_ref[b]
            moved[b] = nb
            pairs.append((b, nb))
        for b in order:
            src_ref[b] = 0
            src_free.append(b)
        for s in seqs:
            self.tables[s] = [moved[b] for b in self.tables[s]]
            if to_cpu:
                self.swapped.add(s)
            else:
                self.swapped.discard(s)
        return pairs

    def swap_out(self, seqs):
        """(device block, host block) pairs; the group's blocks move to the host pool."""
        return self._move(list(seqs), True)

    def swap_in(self, seqs):
        """(host block, device block) pairs; the group comes back to the device."""
        return self._move(list(seqs), False)

    def append_slots(self, seqs):
        """Returns (slots, cow_pairs).  All-or-nothing on a short pool."""
        if len(set(seqs)) != len(seqs) or any(s not in self.tables or s in self.swapped
                                               for s in seqs):
            raise KeyError(seqs)
        # count what the step needs, with reference counts as they will evolve
        refs = {}
        need = 0
        for s in seqs:
            if self.lens[s] % self.block_size == 0:
                need += 1
            else:
                last = self.tables[s][-1]
                r = refs.get(last, self.ref[last])
                if r > 1:
                    need += 1
                    refs[last] = r - 1
        if need > len(self.free):
            raise OutOfBlocks
        slots, pairs = [], []
        for s in seqs:
            pos = self.lens[s]
            table = self.tables[s]
            if pos % self.block_size == 0:
                table.append(self._take())                 # the last block is full
            elif self.ref[table[-1]] > 1:                   # shared: copy on write
                old = table[-1]
                new = self._take()
                self.ref[old] -= 1
                table[-1] = new
                pairs.append((old, new))
            slots.append(table[pos // self.block_size] * self.block_size + pos % self.block_size)
            self.lens[s] = pos + 1
        return slots, pairs
