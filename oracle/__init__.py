"""CPU float64 oracle for the TwoTower denoiser refinement step (test infrastructure only)."""
