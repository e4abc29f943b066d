"""Reference model of the host block manager (test infrastructure).

The pages fix the idea, not a policy:
 * "vLLM — PagedAttention으로 LLM 추론 성능을 2~4배 끌어올린 서빙 엔진" (dev.to),
   section "PagedAttention — OS 가상 메모리에서 영감": blocks are handed out
   only as tokens arrive, free blocks serve any other request, and logical
   blocks map to physical blocks through a per-sequence table.
 * "Nano-vLLM로 배우는 vLLM 추론 엔진 작동 원리 한눈에 정리" (tilnote.io),
   section "KV 캐시와 Block Manager": the block manager keeps block metadata on
   the CPU while the K/V tensors stay on the GPU; prefix blocks can be shared.

The policy modelled here (the library implements the same one, separately):
 * the free blocks form a stack; ``free_order[0]`` is handed out first;
 * a block's reference count is the number of tables that hold it; a block
   returns to the top of the stack when its count reaches zero;
 * releasing a sequence walks its table from logical block 0 upwards;
 * appending a token at position p allocates a block when p % Bs == 0 and
   the token's slot is table[p // Bs] * Bs + p % Bs;
 * a batch append is all-or-nothing: if the free stack cannot cover every new
   block it needs, nothing changes;
 * appending into a block that another table also holds is refused (there is
   no copy-on-write in this policy).
"""
from __future__ import annotations


class OutOfBlocks(RuntimeError):
    pass


class SharedBlockWrite(RuntimeError):
    pass


class BlockManagerModel:
    def __init__(self, num_blocks: int, block_size: int, max_seqs: int, max_blocks_per_seq: int,
                 free_order):
        self.num_blocks = num_blocks
        self.block_size = block_size
        self.max_seqs = max_seqs
        self.max_blocks_per_seq = max_blocks_per_seq
        self.free = [int(b) for b in reversed(list(free_order))]  # top of stack = end of list
        self.ref = [0] * num_blocks
        self.tables = [[] for _ in range(max_seqs)]
        self.lens = [0] * max_seqs
        self.live = [False] * max_seqs

    # -- pool ---------------------------------------------------------------
    def _pop(self) -> int:
        blk = self.free.pop()
        self.ref[blk] = 1
        return blk

    def _release(self, blk: int) -> None:
        self.ref[blk] -= 1
        if self.ref[blk] == 0:
            self.free.append(blk)

    def num_free(self) -> int:
        return len(self.free)

    # -- sequences ----------------------------------------------------------
    def import_seq(self, seq: int, length: int, blocks) -> None:
        """Adopt a sequence whose blocks were laid out outside the free stack."""
        assert not self.live[seq]
        blocks = [int(b) for b in blocks]
        assert len(blocks) == -(-length // self.block_size)
        for blk in blocks:
            self.ref[blk] += 1
        self.tables[seq] = blocks
        self.lens[seq] = length
        self.live[seq] = True

    def add_seq(self, seq: int, length: int) -> None:
        """Admit a sequence of `length` cached tokens into fresh blocks."""
        assert not self.live[seq]
        need = -(-length // self.block_size)
        if need > len(self.free):
            raise OutOfBlocks(seq)
        self.tables[seq] = [self._pop() for _ in range(need)]
        self.lens[seq] = length
        self.live[seq] = True

    def free_seq(self, seq: int) -> None:
        assert self.live[seq]
        for blk in self.tables[seq]:
            self._release(blk)
        self.tables[seq] = []
        self.lens[seq] = 0
        self.live[seq] = False

    def append_tokens(self, seqs) -> list:
        """One new token for each listed sequence; returns the slots."""
        Bs = self.block_size
        need = 0
        for seq in seqs:
            p = self.lens[seq]
            if p % Bs == 0:
                need += 1
            elif self.ref[self.tables[seq][p // Bs]] > 1:
                raise SharedBlockWrite(seq)
        if need > len(self.free):
            raise OutOfBlocks(need)
        slots = []
        for seq in seqs:
            p = self.lens[seq]
            if p % Bs == 0:
                self.tables[seq].append(self._pop())
            slots.append(self.tables[seq][p // Bs] * Bs + p % Bs)
            self.lens[seq] = p + 1
        return slots

    def table_array(self, seq: int):
        row = list(self.tables[seq])
        return row + [-1] * (self.max_blocks_per_seq - len(row))
