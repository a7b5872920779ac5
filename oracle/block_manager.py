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
Slots are physical_block * block_size + offset.
"""
from __future__ import annotations


class OutOfBlocks(Exception):
    pass


class BlockManagerOracle:
    def __init__(self, num_blocks: int, block_size: int):
        self.block_size = block_size
        self.free = list(range(num_blocks - 1, -1, -1))   # pop() gives 0, 1, 2, ...
        self.ref = [0] * num_blocks
        self.tables: dict[int, list[int]] = {}
        self.lens: dict[int, int] = {}

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
        if parent not in self.tables or child in self.tables:
            raise KeyError(child)
        self.tables[child] = list(self.tables[parent])
        self.lens[child] = self.lens[parent]
        for b in self.tables[child]:
            self.ref[b] += 1

    def free_sequence(self, seq: int):
        for b in self.tables.pop(seq):
            self.ref[b] -= 1
            if self.ref[b] == 0:
                self.free.append(b)
        del self.lens[seq]

    def append_slots(self, seqs):
        """Returns (slots, cow_pairs).  All-or-nothing on a short pool."""
        if len(set(seqs)) != len(seqs) or any(s not in self.tables for s in seqs):
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
