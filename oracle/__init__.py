"""CPU oracle for the Sol-Attn forward pass.  TEST INFRASTRUCTURE ONLY (tests, smoke, CPU baseline)."""
